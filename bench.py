#!/usr/bin/env python
"""Benchmark of the sparse MoE feed-forward layer on B200.

One step = one pass of the whole layer (route -> permute -> gate|up grouped GEMM + SwiGLU -> down grouped
GEMM -> weighted combine) over one batch of seeded synthetic tokens, through the library's public API.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]
    python bench.py --kernel gateup|down [--workload NAME] [--shape T=..,E=..] [--gemm FAMILY]

Prints one JSON line (rank 0). Device timing: CUDA events on the launching stream around each step (no events
inside a step), L2 flushed (256 MiB write) before every step outside the events, max over ranks. The per-stage
split comes from a second, separate pass with events between the stages. `e2e` repeats the step with the input
copied from pinned host memory and the output copied back inside the timed region. Multi-GPU runs are
independent replicas (the layer has no cross-GPU exchange): weak scaling, value = all tokens / time.
`--impl reference` times the CPU oracle (plain fp64 C, all host cores) on a bounded token sample.
`--kernel` times one grouped GEMM alone on the workload's realised routing (for profilers); `--shape` shrinks the
workload for such captures and `--gemm` forces a kernel family (single, pair, wide, swap).
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "MoE-layer tokens/s and achieved TFLOP/s or HBM GB/s vs roofline, 1×B200"
DEFAULT_WORKLOAD = "gpt-oss-20b-prefill"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 256 << 20

# DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum) from an ncu capture, keyed by the
# kernel, the workload and a hash of the GEMM sources (comments stripped) at capture time. A stale hash -> null.
# Captured on one launch of the GEMM timed alone on the workload's routing, L2 flushed before it, as the bench
# does before each step:
#   python bench.py --kernel K --workload W --steps 2 --warmup 3 > plain.log 2>&1 &&
#   ncu --metrics dram__bytes_read.sum,dram__bytes_write.sum --clock-control none -k regex:grouped_gemm -s 4 -c 1
#       python bench.py --kernel K --workload W --steps 2 --warmup 3
TRAFFIC = {
    ("grouped_gemm_gateup", "gpt-oss-20b-prefill", "e1c4dc9759352dbe"): 1248905472,
    ("grouped_gemm_down", "gpt-oss-20b-prefill", "e1c4dc9759352dbe"): 713312000,
    ("grouped_gemm_gateup", "mixtral-8x7b-prefill", "e1c4dc9759352dbe"): 2874045952,
    ("grouped_gemm_down", "mixtral-8x7b-prefill", "e1c4dc9759352dbe"): 2457829376,
    ("grouped_gemm_gateup", "zipf-128e", "e1c4dc9759352dbe"): 1593265664,
    ("grouped_gemm_down", "zipf-128e", "e1c4dc9759352dbe"): 1083839744,
    ("grouped_gemm_gateup", "decode-256e-shared", "e1c4dc9759352dbe"): 12932052992,
    ("grouped_gemm_down", "decode-256e-shared", "e1c4dc9759352dbe"): 6467805184,
    ("grouped_gemm_gateup", "decode-256e-shared-mxfp4", "e1c4dc9759352dbe"): 3671495936,
    ("grouped_gemm_down", "decode-256e-shared-mxfp4", "e1c4dc9759352dbe"): 1772047616,
}
KERNEL_SOURCES = ["mixture_experts_ffn_11_b200/csrc/" + f for f in
                  ("gemm.cuh", "gemm_pair.cuh", "gemm_wide.cuh", "gemm_swap.cuh", "gemm_fp4.cuh", "gemm_fp4_mma.cuh",
                   "sm100.cuh", "common.cuh", "moe.cu")]


def kernel_source_hash() -> str:
    """Hash of the GEMM sources with comments and blank lines removed (a comment edit keeps the figures)."""
    import re

    h = hashlib.sha256()
    for p in KERNEL_SOURCES:
        src = open(os.path.join(ROOT, p)).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        lines = (re.sub(r"//.*$", "", ln).rstrip() for ln in src.splitlines())
        h.update("\n".join(ln for ln in lines if ln).encode())
    return h.hexdigest()[:16]


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        p = json.load(open(path))
        return {k: float(p[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--cpu-seconds", type=float, default=15.0, help="target CPU time of the oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--settle-seconds", type=float, default=2.0,
                    help="extra untimed load after the warm-up so clocks and power settle")
    ap.add_argument("--kernel", choices=["gateup", "down"], default=None,
                    help="time one grouped GEMM alone (kernel-only mode, for profilers)")
    ap.add_argument("--gemm", choices=["auto", "single", "pair", "wide", "swap"], default="auto",
                    help="force a grouped-GEMM kernel family")
    ap.add_argument("--dispatch", choices=["fused", "separate"], default="separate",
                    help="prefill: row gather and combine as their own kernels (default), or inside the grouped GEMMs")
    ap.add_argument("--shape", default="", help="comma-separated workload overrides, e.g. T=1024,E=64 (profiling)")
    ap.add_argument("--backward", action="store_true",
                    help="time the training step: forward + backward with weight gradients (not the headline)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    return args


# ---- distributed plumbing (replicas) ----------------------------------------------------------------

def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)), int(os.environ.get("WORLD_SIZE", 1))


def dist_init(backend: str):
    import torch.distributed as dist

    rank, local, world = dist_env()
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return rank, local, world


def barrier(device=None):
    import torch.distributed as dist

    if dist.is_available() and dist.is_initialized():
        if device is not None and dist.get_backend() == "nccl":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def max_over_ranks(value: float, device=None) -> float:
    """Max of a float over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()):
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device if dist.get_backend() == "nccl" else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---- clocks ------------------------------------------------------------------------------------------

class ClockSampler:
    """nvidia-smi samples of SM clock, power and throttle reasons for one GPU while the benchmark runs."""

    FIELDS = ["timestamp", "uuid", "clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.active",
              "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]

    def __init__(self, uuid: str | None):
        self.uuid = uuid
        self.proc = None
        self.out = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "--query-gpu=" + ",".join(self.FIELDS),
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=self.out, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        self.out.flush()

    def summary(self, t0: float, t1: float) -> dict:
        rows = []
        self.out.seek(0)
        for line in self.out.read().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) != len(self.FIELDS):
                continue
            if self.uuid and self.uuid not in parts[1]:
                continue
            try:
                ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                rows.append((ts, float(parts[2]), float(parts[3]), parts[4], parts[6:]))
            except ValueError:
                continue
        inside = [r for r in rows if t0 <= r[0] <= t1]
        window = "timed region"
        if len(inside) < 3:  # short timed region: include the preceding second of the same load (warm-up)
            inside = [r for r in rows if t0 - 1.0 <= r[0] <= t1]
            window = "timed region + preceding 1 s of identical warm-up load"
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in inside for i, v in enumerate(r[4]) if v.lower().startswith("active")})
        powers = [float(r[3]) for r in inside if r[3].replace(".", "", 1).isdigit()]
        return {"sm_mhz": statistics.median(r[1] for r in inside), "sm_max_mhz": max(r[2] for r in inside),
                "reasons": reasons, "samples": len(inside), "window": window,
                "power_w_max": max(powers) if powers else None}


# ---- roofline arithmetic -------------------------------------------------------------------------------

def weight_bytes(wl) -> float:
    """Bytes per expert weight: 2 for bf16; MXFP4 stores a 4-bit code plus one 8-bit scale per 32 weights."""
    return 0.5 + 1.0 / 32 if wl.weights == "mxfp4" else 2.0


def gemm_figures(wl, counts, folded_shared=False):
    """Algorithmic FLOPs and DRAM bytes per launch of the two grouped GEMMs, from the realised routing; with
    folded_shared the launches also compute the shared expert (as wide as a routed one) as one more group of T
    rows."""
    R, d, f, wb = wl.R, wl.d, wl.f, weight_bytes(wl)
    active = int((counts > 0).sum())
    groups, rows = active + (1 if folded_shared else 0), R + (wl.T if folded_shared else 0)
    gateup = {"flop": 4.0 * rows * d * f, "bytes": groups * 2 * f * d * wb + rows * d * 2 + rows * f * 2}
    down = {"flop": 2.0 * rows * f * d, "bytes": groups * d * f * wb + rows * f * 2 + rows * d * 2}
    return active, gateup, down


def layer_figures(wl, active):
    flop = wl.flops()
    wb = weight_bytes(wl)
    bytes_ = (active * 3 * wl.d * wl.f * wb + 3 * wl.d * wl.shared_f * wb + wl.T * wl.d * 2 * 2 + wl.E * wl.d * 4)
    return flop, bytes_


def roofline_entry(name, fig, t_ms, peaks, peak_kind, traffic_bytes):
    t_flop = fig["flop"] / (peaks[peak_kind] * 1e12)
    t_byte = fig["bytes"] / (peaks["hbm_gbs"] * 1e9)
    if t_flop >= t_byte:
        achieved = fig["flop"] / (t_ms * 1e-3) / 1e12
        return {"kernel": name, "bound": "tensor", "achieved": round(achieved, 2), "peak": peaks[peak_kind],
                "unit": "TFLOP/s", "frac": round(achieved / peaks[peak_kind], 4), "traffic": traffic_bytes,
                "algorithmic_flop": fig["flop"], "algorithmic_bytes": fig["bytes"], "launch_ms": round(t_ms, 5)}
    achieved = fig["bytes"] / (t_ms * 1e-3) / 1e9
    return {"kernel": name, "bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"],
            "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4), "traffic": traffic_bytes,
            "algorithmic_flop": fig["flop"], "algorithmic_bytes": fig["bytes"], "launch_ms": round(t_ms, 5)}


# ---- CPU oracle (baseline and reference arm) ------------------------------------------------------------

class OracleStep:
    """One pass of the oracle over a token sample: router logits, top-k, grouping, per-token expert loop."""

    def __init__(self, wl):
        import numpy as np

        import oracle
        import synth

        self.np, self.oracle, self.wl = np, oracle, wl
        self.x = synth.x_host(wl)
        self.wr = synth.w_router_host(wl)
        self.bias = synth.zipf_bias(wl)
        self.order = np.random.default_rng(1234).permutation(wl.T).astype(np.int32)
        self.gu = [None] * wl.E
        self.dn = [None] * wl.E
        # MXFP4 workloads compute with the weights the encoding represents
        self.enc = (lambda a: oracle.mxfp4_round_trip(a)) if wl.weights == "mxfp4" else (lambda a: a)
        self.shared = tuple(self.enc(a) for a in synth.shared_host(wl)) if wl.shared_f else (None, None)
        self.threads = max(1, len(os.sched_getaffinity(0)))

    def prepare(self, n):
        """Generate the experts the first n sampled tokens select (outside any timing)."""
        import synth

        toks = self.order[:n]
        l = self.oracle.router_logits(self.x[toks], self.wr, self.bias).astype(self.np.float32)
        idx, _ = self.oracle.topk(l, self.wl.k, self.wl.route)
        for e in self.np.unique(idx):
            if self.gu[e] is None:
                self.gu[e] = self.enc(synth.w_gateup_expert_host(self.wl, int(e)))
                self.dn[e] = self.enc(synth.w_down_expert_host(self.wl, int(e)))

    def run(self, n):
        o, np = self.oracle, self.np
        xs = self.x[self.order[:n]]
        l64 = o.router_logits(xs, self.wr, self.bias)
        idx, w = o.topk(l64.astype(np.float32), self.wl.k, self.wl.route)
        o.permute(idx, self.wl.E)
        return o.moe_tokens(xs, self.gu, self.dn, idx, w, np.arange(n, dtype=np.int32), self.shared[0],
                            self.shared[1], nthreads=self.threads)


def calibrate_sample(step: OracleStep, seconds: float, cap: int) -> int:
    n0 = min(64, cap)  # enough tokens to keep every host thread busy, so the per-token time is representative
    step.prepare(n0)
    t = time.perf_counter()
    step.run(n0)
    per_tok = max((time.perf_counter() - t) / n0, 1e-6)
    return int(max(1, min(cap, seconds / per_tok)))


def cpu_baseline(wl, seconds: float) -> dict:
    step = OracleStep(wl)
    n = calibrate_sample(step, seconds, wl.T)
    step.prepare(n)
    t = time.perf_counter()
    step.run(n)
    dt = time.perf_counter() - t
    return {"value": round(n / dt, 3), "unit": "tokens/s", "cores": step.threads, "kind": "oracle",
            "sample": f"{n} of the {wl.T} tokens (seeded sample), whole layer per token in fp64 "
                      f"(router, top-k, grouping, per-token expert loop), {dt:.1f} s wall"}


def workload_config(wl) -> dict:
    return {"workload": wl.name, "T": wl.T, "d": wl.d, "f": wl.f, "E": wl.E, "k": wl.k, "route": wl.route,
            "shared_f": wl.shared_f, "zipf_s": wl.zipf_s, "seed": wl.seed, "expert_weights": wl.weights,
            "l2": "flushed (256 MiB write) before every timed step, outside the events"}


DATA = "synthetic: seeded generator, x ~N(0,1) bf16, weights ~N(0,0.02) (random init, no checkpoint)"


def run_reference(args):
    import synth

    rank, _, world = dist_env()
    if rank != 0:
        return 0
    wl = synth.workload(args.workload)
    step = OracleStep(wl)
    budget = 150.0 / max(1, args.steps + args.warmup)  # whole run within a few minutes
    n = calibrate_sample(step, budget, wl.T)
    step.prepare(n)
    for _ in range(args.warmup):
        step.run(n)
    times = []
    for _ in range(args.steps):
        t = time.perf_counter()
        step.run(n)
        times.append(time.perf_counter() - t)
    ms = 1e3 * sum(times) / len(times)
    value = n / (ms * 1e-3)
    sample = f"{n} of the {wl.T} tokens per step (seeded sample); oracle in fp64 on {step.threads} host threads"
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": DATA, "config": workload_config(wl),
            "cpu_baseline": {"value": round(value, 3), "unit": "tokens/s", "cores": step.threads, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---- our arm --------------------------------------------------------------------------------------------

def bench_workload(args):
    """The workload named by --workload, with any --shape overrides (a renamed copy, never the headline)."""
    import synth

    wl = synth.workload(args.workload)
    if args.shape:
        over = {}
        for item in args.shape.split(","):
            key, val = item.split("=")
            if key not in ("T", "d", "f", "E", "k", "shared_f"):
                raise SystemExit(f"--shape: {key} cannot be overridden")
            over[key] = int(val)
        tag = ",".join(f"{k}={v}" for k, v in over.items())
        wl = synth.workload(args.workload, **over)
        wl = synth.Workload(**{**wl.__dict__, "name": f"{wl.name}[{tag}]"})
    return wl


def setup_layer(args, dev):
    import torch

    import synth
    from mixture_experts_ffn_11_b200 import MoEFFN

    wl = bench_workload(args)
    synth.build_cuda()
    inp = synth.device_inputs(wl, dev)
    # a forced kernel family applies to the grouped-copy path only
    fuse = args.dispatch == "fused" and args.gemm in ("auto", "swap")
    layer = MoEFFN(inp["w_router"], inp["w_gateup"], inp["w_down"], wl.k, wl.route, inp["bias"],
                   inp["w_gateup_shared"], inp["w_down_shared"], weights=wl.weights, fused=fuse)
    if wl.weights != "bf16":  # the layer keeps only its encoded weights
        for key in ("w_gateup", "w_down", "w_gateup_shared", "w_down_shared"):
            inp[key] = None
        torch.cuda.empty_cache()
    return wl, inp, layer


def run_kernel(args):
    """One grouped GEMM alone, on the routing the layer realises: W warm-up launches, then K launches each after
    an L2 flush, CUDA events around each launch. For profilers (select the kernel with -k and skip the warm-up
    launches) and for comparing kernel families."""
    import torch

    from mixture_experts_ffn_11_b200 import _native as N

    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    N.set_gemm_kernel(args.gemm)
    wl, inp, layer = setup_layer(args, dev)
    layer.forward(inp["x"])
    b = layer.buf
    s = torch.cuda.current_stream(dev)
    if args.kernel == "gateup" and layer._fused(wl.T):
        launch = lambda: N.grouped_gemm_gateup_gather(inp["x"], b["perm_src"], layer.w_gateup, b["offsets"],  # noqa
                                                      b["h"], None, s)
    elif args.kernel == "gateup":
        launch = lambda: layer.routed_gateup(b, s)  # noqa: E731
    else:
        launch = lambda: layer.routed_down(b, s)  # noqa: E731
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    for _ in range(args.warmup):
        flush.zero_()
        launch()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for a, c in ev:
        flush.zero_()
        a.record(s)
        launch()
        c.record(s)
    torch.cuda.synchronize(dev)
    if N.get_device_error():
        raise SystemExit("device error word set")
    ms = statistics.mean(a.elapsed_time(c) for a, c in ev)
    counts = b["counts"].cpu().numpy()
    active, fig_gu, fig_dn = gemm_figures(wl, counts, layer._fold(wl.T))
    peaks, src = load_peaks()
    fig = fig_gu if args.kernel == "gateup" else fig_dn
    roof = roofline_entry(f"grouped_gemm_{args.kernel}", fig, ms, peaks, "bf16_tflops", None)
    roof["peak_source"] = f"{src} {'hbm_gbs' if roof['bound'] == 'hbm' else 'bf16_tflops'}"
    print(json.dumps({"kernel_only": args.kernel, "gemm_family": args.gemm, "ms": round(ms, 5), "launches": args.steps,
                      "config": workload_config(wl), "active_experts": active, "roofline": roof}), flush=True)
    return 0


def run_ours(args):
    import torch

    import synth
    from mixture_experts_ffn_11_b200 import _native as N
    from mixture_experts_ffn_11_b200 import get_device_error

    rank, local, world = dist_init("nccl")
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA GPU (there is no CPU fallback)")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    N.set_gemm_kernel(args.gemm)
    wl, inp, layer = setup_layer(args, dev)
    x = inp["x"]
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    launches_per_step = layer.kernel_launches(wl.T, train=args.backward)
    sampler = ClockSampler(torch.cuda.get_device_properties(dev).uuid.__str__() if rank >= 0 else None)
    sampler.start()

    dy = None
    if args.backward:
        dy = torch.empty(wl.T, wl.d, dtype=torch.bfloat16, device=dev)
        synth.fill_device(dy, wl.seed, synth.TID_DY, 0, synth.X_SIGMA)
        launches_per_step += layer.backward_kernel_launches(wl.T, train_forward=True)

    def step(timing=None):
        y = layer.forward(x, timing=timing, train=dy is not None)
        if dy is not None:
            layer.backward(dy, timing=timing)
        return y

    # warm-up: W steps, then keep the same load going for ~2 s so clocks and power settle
    for _ in range(args.warmup):
        flush.zero_()
        step()
    t_end = time.perf_counter() + args.settle_seconds
    while time.perf_counter() < t_end:
        flush.zero_()
        step()
        torch.cuda.synchronize(dev)
    torch.cuda.synchronize(dev)
    if get_device_error():
        raise SystemExit("device error word set during warm-up")

    def timed_pass(stage_events: bool):
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
        stage_ev = [dict() for _ in range(K)]
        barrier(dev)
        torch.cuda.synchronize(dev)
        t_a = time.time()
        for i in range(K):
            flush.zero_()
            ev[i][0].record(stream)
            step(timing=stage_ev[i] if stage_events else None)
            ev[i][1].record(stream)
        torch.cuda.synchronize(dev)
        barrier(dev)
        t_b = time.time()
        step_ms = [a.elapsed_time(b) for a, b in ev]
        stages = {}
        if stage_events:
            for name in stage_ev[0]:
                stages[name] = statistics.mean(a.elapsed_time(b) for a, b in (s[name] for s in stage_ev))
        return step_ms, stages, t_a, t_b

    # headline: K steps with events only around each whole step
    K = args.steps
    step_ms, _, t0, t1 = timed_pass(False)
    total_ms = max_over_ranks(sum(step_ms), dev)
    ms_per_step = total_ms / K
    err = get_device_error()
    if err:
        raise SystemExit(f"device error word {err:#x} set during the timed region")
    # breakdown: a second pass of K steps with events between the stages (they split the programmatic launch
    # overlap between kernels, so this pass runs a little slower than the headline; both are reported)
    staged_ms, stages, _, _ = timed_pass(True)
    staged_ms_per_step = max_over_ranks(sum(staged_ms), dev) / K

    # end to end, as a server would run it: every step copies its input from pinned host memory and its
    # output back to pinned host memory, on their own streams, so step i's copies overlap the layer of the
    # neighbouring steps. Two buffer sets (layer objects sharing the weights) alternate; events order every
    # reuse of a buffer after the last reader of its previous contents.
    e2e = None
    if not args.no_e2e and not args.backward:
        layers = [layer, layer.sibling()]
        x_host = [x.cpu().pin_memory() for _ in range(2)]
        y_host = [torch.empty(wl.T, wl.d, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
        x_dev = [torch.empty_like(x) for _ in range(2)]
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        s_comp = stream

        def run_e2e(n):
            ev_in = [torch.cuda.Event() for _ in range(n)]
            ev_done = [torch.cuda.Event() for _ in range(n)]
            ev_out = [torch.cuda.Event() for _ in range(n)]
            for i in range(n):
                b = i & 1
                with torch.cuda.stream(s_in):
                    if i >= 2:
                        s_in.wait_event(ev_done[i - 2])  # x_dev[b] no longer read by step i-2
                    x_dev[b].copy_(x_host[b], non_blocking=True)
                    ev_in[i].record(s_in)
                s_comp.wait_event(ev_in[i])
                if i >= 2:
                    s_comp.wait_event(ev_out[i - 2])  # step i-2's output copied out of layers[b]
                y = layers[b].forward(x_dev[b], stream=s_comp)
                ev_done[i].record(s_comp)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(ev_done[i])
                    y_host[b].copy_(y, non_blocking=True)
                    ev_out[i].record(s_out)
            return ev_out[-1]

        run_e2e(max(args.warmup, 2))
        torch.cuda.synchronize(dev)
        barrier(dev)
        torch.cuda.synchronize(dev)
        e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e_start.record(s_in)
        last = run_e2e(K)
        s_out.wait_event(last)
        e_end.record(s_out)
        torch.cuda.synchronize(dev)
        barrier(dev)
        e2e_ms = max_over_ranks(e_start.elapsed_time(e_end), dev) / K
        nbytes = wl.T * wl.d * 2
        e2e = {"value": round(world * wl.T / (e2e_ms * 1e-3), 1), "unit": "tokens/s", "ms_per_step": round(e2e_ms, 4),
               "h2d_bytes_per_step": nbytes, "d2h_bytes_per_step": nbytes,
               "path": "pinned host x -> device on a copy stream, MoEFFN.forward on the compute stream, device y -> "
                       "pinned host on a second copy stream; two buffer sets, copies of one step overlap the layer "
                       "of the next",
               "l2": "not flushed (steps overlap); each step streams its expert weights (larger than L2) and a "
                     "fresh input from the host",
               "comparable_with_value": False}
    sampler.stop()
    clocks = sampler.summary(t0, t1)

    counts = layer.buf["counts"].cpu().numpy()
    active, fig_gu, fig_dn = gemm_figures(wl, counts, layer._fold(wl.T))
    peaks, peak_src = load_peaks()
    peak_kind = "bf16_tflops_sustained" if total_ms > 1000.0 else "bf16_tflops"
    src_hash = kernel_source_hash()
    tr = TRAFFIC.get(("grouped_gemm_gateup", wl.name, src_hash))
    roof = roofline_entry("grouped_gemm_gateup", fig_gu, stages["gateup"], peaks, peak_kind, tr)
    roof["peak_source"] = f"{peak_src} {'hbm_gbs' if roof['bound'] == 'hbm' else peak_kind}"
    roof["launch_ms_source"] = "CUDA events around the kernel in the breakdown pass (not the headline pass)"
    roof_dn = roofline_entry("grouped_gemm_down", fig_dn, stages["down"], peaks, peak_kind,
                             TRAFFIC.get(("grouped_gemm_down", wl.name, src_hash)))
    lflop, lbytes = layer_figures(wl, active)
    t_roof = max(lflop / (peaks[peak_kind] * 1e12), lbytes / (peaks["hbm_gbs"] * 1e9))
    line = {"metric": METRIC, "value": round(world * wl.T / (ms_per_step * 1e-3), 1), "unit": "tokens/s",
            "n_gpus": world, "steps": K, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": DATA,
            "config": workload_config(wl), "roofline": roof, "roofline_down": roof_dn,
            "layer_roofline": {"flop": lflop, "bytes": lbytes, "active_experts": active,
                               "t_roofline_ms": round(t_roof * 1e3, 5),
                               "frac": round(t_roof * 1e3 / ms_per_step, 4),
                               "achieved_tflops": round(lflop / (ms_per_step * 1e-3) / 1e12, 2)},
            "breakdown_ms": {k: round(v, 5) for k, v in stages.items()},
            "breakdown_pass_ms_per_step": round(staged_ms_per_step, 5),
            "gpu_launches": K * launches_per_step, "clocks": clocks, "e2e": e2e,
            "parallelism": "replicas" if world > 1 else "single GPU"}
    if args.gemm != "auto":
        line["gemm_family"] = args.gemm
    line["config"]["dispatch"] = ("gather in gate|up GEMM, combine in down GEMM" if layer._fused(wl.T)
                                  else "moe_permute gather, moe_unpermute_combine")
    if args.backward:
        # the training step: forward (keeping the gate|up pre-activations) + backward (top-k selection held
        # fixed), weight gradients included: 6 + 12 R d f, and the same for the shared expert over T rows
        R, d, f, fs = wl.R, wl.d, wl.f, wl.shared_f
        bwd_flop = {"bwd_dh": 2.0 * R * d * f, "bwd_dx_perm": 4.0 * R * d * f,
                    "bwd_dw_down": 2.0 * R * d * f, "bwd_dw_gateup": 4.0 * R * d * f}
        train_flop = lflop + 12.0 * R * d * f + 12.0 * wl.T * d * fs
        top = max(bwd_flop, key=lambda n: stages[n])  # the backward stage that takes longest
        tr_roof = roofline_entry(top, {"flop": bwd_flop[top], "bytes": 0.0}, stages[top], peaks, peak_kind, None)
        line.update({"metric": "MoE-layer training step (forward + backward) tokens/s and TFLOP/s, 1xB200",
                     "training_step": {"flop": train_flop,
                                       "achieved_tflops": round(train_flop / (ms_per_step * 1e-3) / 1e12, 2),
                                       "frac_of_peak": round(train_flop / (ms_per_step * 1e-3) / 1e12 /
                                                             peaks[peak_kind], 4)},
                     "roofline_backward": tr_roof,
                     "roofline_backward_all": {n: roofline_entry(n, {"flop": fl, "bytes": 0.0}, stages[n], peaks,
                                                                 peak_kind, None)["frac"]
                                               for n, fl in bwd_flop.items()}})
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not args.backward:
        line["cpu_baseline"] = cpu_baseline(wl, args.cpu_seconds)
    if rank == 0:
        print(json.dumps(line), flush=True)
    import torch.distributed as dist

    if dist.is_available() and dist.is_initialized():
        dist.destroy_process_group()
    return 0


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    if args.kernel:
        return run_kernel(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
