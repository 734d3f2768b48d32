#!/usr/bin/env python
"""Throughput of one top-k MoE SwiGLU layer forward on B200 GPUs.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl ours|reference]

One step = one whole layer call (router, permutation, grouped gate_up + SwiGLU, grouped
down + weighted combine, shared expert when the layer has one, bf16 output) over one batch
of synthetic tokens already resident in HBM.  The call is captured once in a CUDA graph
and every step replays it; L2 is flushed (a 512 MiB write, then a 512 MiB read) before
every timed step, outside the timed interval, and each step is timed with CUDA events on
the launching stream.

Default run (N = 1): the headline workload is the fine-grained layer with a shared expert
(T=4096, D=4096, E=512, K=10, f=1024, f_s=1024), timed over exactly --steps steps; a
``per_config`` object then measures every other workload (tiny, decode with natural and
concentrated routing, prefill, the Zipf sweep T in {1, 16, 128, 1024, 16384}) as the
median of >= 50 cold-L2 graph replays, with a hot-L2 median beside it, per-kernel times,
clocks and the CPU oracle timed on a bounded sample of the same workload.

With --gpus N > 1 every rank (one process per GPU, launched by torchrun, or by this script
itself when WORLD_SIZE is not set) runs an independent replica of the batch (no
exchange): the reported value is all ranks' tokens over the slowest rank's time.

``--impl reference`` times the CPU oracle (fp64, OpenMP) on this host instead.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import re
import socket
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE layer tokens/s on 1 B200 and % of roofline (HBM GB/s or bf16 TC util)"
UNIT = "tokens/s"
HEADLINE = "finegrained"
PER_CONFIG = ("tiny", "decode", "decode_concentrated", "prefill", "zipf@T1", "zipf@T16",
              "zipf@T128", "zipf@T1024", "zipf@T16384")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# B200 data-sheet figures, for context beside the measured peaks
NOMINAL_PEAKS = {"hbm_gbs": 8000.0, "bf16_tflops": 2250.0}
FLUSH_BYTES = 512 << 20
PROFILE_DIR = os.path.join(ROOT, "profiles")


# ---------------------------------------------------------------- accounting


def describe(cfg) -> str:
    s = f"{cfg.name}: T={cfg.T} D={cfg.D} E={cfg.E} K={cfg.K} f={cfg.f}"
    if cfg.f_s:
        s += f" f_s={cfg.f_s}"
    return s + f" routing={cfg.routing}"


def layer_flops(cfg) -> float:
    """2*3*D*f per routed (token, expert) row, 2*3*D*f_s per token for the shared expert,
    plus the router's 2*D*E per token."""
    return 6.0 * cfg.D * cfg.f * cfg.T * cfg.K + 6.0 * cfg.D * cfg.f_s * cfg.T + \
        2.0 * cfg.T * cfg.D * cfg.E


def layer_bytes(cfg, U: int) -> float:
    """bf16 weights of the U experts hit (+ shared, + router), x in, y out."""
    return 2.0 * 3 * cfg.D * cfg.f * U + 2.0 * 3 * cfg.D * cfg.f_s + 2.0 * cfg.E * cfg.D + \
        4.0 * cfg.T * cfg.D


def gate_up_bytes(cfg, U: int) -> float:
    """Algorithmic bytes of one grouped gate_up launch: gate+up weights of the U experts
    hit, the T*K gathered token rows read, the T*K x f SwiGLU rows written."""
    rows = cfg.T * cfg.K
    return 2.0 * 2 * cfg.D * cfg.f * U + 2.0 * rows * cfg.D + 2.0 * rows * cfg.f


def gate_up_flops(cfg) -> float:
    return 4.0 * cfg.D * cfg.f * cfg.T * cfg.K


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            d = json.load(fh)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def layer_roofline(cfg, U: int, ms: float, peaks: dict, src: str) -> dict:
    """The layer against max(F / P_tensor, B / BW_hbm): with the measured burst tensor peak
    (the step is milliseconds long, not a seconds-long power-capped loop), the sustained one
    beside it, and the data-sheet figures for context."""
    F, B = layer_flops(cfg), layer_bytes(cfg, U)
    bw = peaks["hbm_gbs"] * 1e9
    burst = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]) * 1e12
    sust = peaks.get("bf16_tflops_sustained", burst / 1e12) * 1e12
    t_burst = max(F / burst, B / bw)
    t_sust = max(F / sust, B / bw)
    t_nom = max(F / (NOMINAL_PEAKS["bf16_tflops"] * 1e12), B / (NOMINAL_PEAKS["hbm_gbs"] * 1e9))
    s = ms / 1e3
    return {
        "bound": "tensor" if F / burst > B / bw else "hbm",
        "flops": F, "bytes": B,
        "t_roof_ms": 1e3 * t_burst, "frac": t_burst / s,
        "t_roof_ms_sustained": 1e3 * t_sust, "frac_sustained": t_sust / s,
        "frac_nominal": t_nom / s,
        "achieved_tflops": F / s / 1e12, "achieved_gbs": B / s / 1e9,
        "peaks": f"{src}: {burst / 1e12:.1f} TFLOP/s burst (bf16_tflops), "
                 f"{sust / 1e12:.1f} sustained, {bw / 1e9:.1f} GB/s (hbm_gbs); nominal "
                 f"{NOMINAL_PEAKS['bf16_tflops']:.0f} TFLOP/s, {NOMINAL_PEAKS['hbm_gbs']:.0f} GB/s",
    }


def _code_only(text: str) -> str:
    """C/C++ source without comments and with whitespace collapsed: an edit to a comment
    does not change the kernel the profiler measured."""
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


def kernel_source_hash() -> str:
    """Identifies the grouped GEMM kernels' source (code only) that a profile was taken on."""
    h = hashlib.sha256()
    for f in ("grouped_gemm.cu", "ptx.cuh", "common.cuh"):
        with open(os.path.join(ROOT, "top_routing_grouped_03_b200", "csrc", f), encoding="utf-8") as fh:
            h.update(_code_only(fh.read()).encode("utf-8"))
    return h.hexdigest()[:16]


def ncu_traffic(kernel: str, workload: str):
    """dram read+write bytes per launch from the committed ncu summary of this kernel and
    workload, or None when absent or taken on a different kernel source."""
    path = os.path.join(PROFILE_DIR, f"{kernel}_{workload}.md")
    if not os.path.exists(path):
        return None
    vals = {}
    with open(path, encoding="utf-8") as fh:
        for line in fh:
            if line.startswith("- ") and ":" in line:
                k, v = line[2:].split(":", 1)
                vals[k.strip()] = v.strip().strip("`")
    if vals.get("kernel_source_sha256") != kernel_source_hash():
        return None
    try:
        return float(vals["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


# ---------------------------------------------------------------- ranks


def max_over_ranks(x: float, device=None) -> float:
    """The slowest rank's figure (all-reduce MAX); x itself without a process group."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(world: int, tokens_per_rank: int, steps: int, slowest_ms: float) -> float:
    """Tokens of all ranks over the slowest rank's device time, per second."""
    return world * tokens_per_rank * steps / (slowest_ms / 1e3)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def launch_ranks(nproc: int, argv) -> int:
    """Run this script as `nproc` ranks of one node under torchrun (rendezvous on
    127.0.0.1) and return its exit status; the ranks read RANK/WORLD_SIZE/LOCAL_RANK."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           f"--nproc-per-node={nproc}", "--master-addr", "127.0.0.1",
           f"--master-port={_free_port()}", os.path.abspath(__file__), *argv]
    return subprocess.call(cmd)


def rank_env():
    """(rank, world, local_rank) from the launcher's environment, or (0, 1, 0)."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


# ---------------------------------------------------------------- clocks


class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.tmp = None

    def start(self):
        self.tmp = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu_id}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=self.tmp, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.25)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.1)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.tmp.flush()
        self.tmp.seek(0)
        rows = [l.strip().split(", ") for l in self.tmp.read().splitlines() if l.strip()]
        self.tmp.close()
        os.unlink(self.tmp.name)
        sm, smax, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for r in rows:
            if len(r) < 9:
                continue
            try:
                sm.append(float(r[1]))
                smax.append(float(r[2]))
            except ValueError:
                continue
            for n, v in zip(names, r[5:9]):
                if v.strip().lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax),
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------- CPU oracle


def cpu_sample_tokens(cfg) -> int:
    """Tokens the CPU oracle takes per pass: the whole batch of the small layers, a few
    tokens of the multi-GB ones (a pass then takes about a second on 16 cores)."""
    per_token_flops = 6.0 * cfg.D * (cfg.f * cfg.K + cfg.f_s) + 2.0 * cfg.D * cfg.E
    return int(max(1, min(cfg.T, 64, 3.0e9 // per_token_flops)))


class OracleSample:
    """The oracle's inputs for the first n tokens of a layer: x rows, the router weight and
    only the experts those tokens route to (copied to the host once, outside any timing)."""

    def __init__(self, inp, n: int):
        import numpy as np
        import torch

        import oracle
        self.oracle = oracle
        oracle.build()
        cfg = inp.cfg
        self.n = n
        self.K = cfg.K
        self.x = inp.x[:n].cpu()
        self.w_router = inp.w_router.cpu()
        self.logit_bias = None if inp.logit_bias is None else inp.logit_bias.cpu()
        self.w_shared_gate = None if inp.w_shared_gate is None else inp.w_shared_gate.cpu()
        r = oracle.route(self.x, self.w_router, cfg.K, self.logit_bias, self.w_shared_gate)
        self.experts = np.unique(r["idx"])
        ex = torch.as_tensor(self.experts.astype(np.int64), device=inp.w_gate_up.device)
        self.w_gate_up = inp.w_gate_up.index_select(0, ex).cpu()
        self.w_down = inp.w_down.index_select(0, ex).cpu()
        self.lookup = np.full(cfg.E, -1, np.int32)
        self.lookup[self.experts] = np.arange(len(self.experts), dtype=np.int32)
        self.w_shared_gate_up = None if inp.w_shared_gate_up is None else inp.w_shared_gate_up.cpu()
        self.w_shared_down = None if inp.w_shared_down is None else inp.w_shared_down.cpu()

    def step(self) -> int:
        """One pass: route the sampled tokens and sum their experts, fp64."""
        o = self.oracle
        r = o.route(self.x, self.w_router, self.K, self.logit_bias, self.w_shared_gate)
        o.experts(self.x, self.lookup[r["idx"]], r["alpha"], self.w_gate_up, self.w_down, None,
                  self.w_shared_gate_up, self.w_shared_down, r["shared_gate"])
        return self.n


def cpu_baseline(inp, budget_s: float) -> dict:
    """The oracle as it stands on this host's cores over a bounded sample of the workload:
    the first n tokens (router + expert sum), repeated until about budget_s of work."""
    cfg = inp.cfg
    s = OracleSample(inp, cpu_sample_tokens(cfg))
    n, reps, t0 = 0, 0, time.perf_counter()
    while True:
        n += s.step()
        reps += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    dt = time.perf_counter() - t0
    return {"value": n / dt, "unit": UNIT, "cores": int(os.environ.get("OMP_NUM_THREADS", "1")),
            "kind": "oracle",
            "sample": f"the first {s.n} of {cfg.T} tokens (router + expert sum over their "
                      f"{len(s.experts)} experts, fp64) x {reps} passes, {dt:.1f} s"}


def run_reference(args, cfg, world, rank):
    """The oracle on the host cores, on the workload of our arm, bounded per step."""
    if rank != 0:
        return 0
    import workloads
    dev = "cuda" if _cuda_ok() and big_layer(cfg) else "cpu"
    inp = workloads.make_inputs(cfg, device=dev)
    s = OracleSample(inp, 1)
    t1 = time.perf_counter()
    s.step()
    per_tok = max(time.perf_counter() - t1, 1e-3)
    budget = 90.0  # seconds for the whole warmup + timed run
    ntok = int(max(1, min(cfg.T, 64, budget / (args.steps + args.warmup) / per_tok)))
    s = OracleSample(inp, ntok)
    for _ in range(args.warmup):
        s.step()
    t0 = time.perf_counter()
    n = 0
    for _ in range(args.steps):
        n += s.step()
    dt = time.perf_counter() - t0
    value = n / dt
    cores = int(os.environ.get("OMP_NUM_THREADS", "1"))
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * dt / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": describe(cfg), "tokens_per_step": ntok},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"the first {ntok} of {cfg.T} tokens per step (router + "
                                   f"expert sum), fp64"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def _cuda_ok() -> bool:
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


def big_layer(cfg) -> bool:
    """Layers whose weights are drawn on the GPU (multi-GB; same recipe, CUDA generator)."""
    return 3 * cfg.E * cfg.D * cfg.f + cfg.T * cfg.D > (1 << 28)


# ---------------------------------------------------------------- GPU arm


class Bench:
    """Timing helpers on one device: the L2 flush, the graph of one layer call, events."""

    def __init__(self, dev, flush_mib: int):
        import torch
        self.torch = torch
        self.dev = dev
        self.flush_mib = flush_mib
        n = max(flush_mib, 1) << 20
        self.flush_w = torch.empty(n, dtype=torch.uint8, device=dev)
        self.flush_r = torch.ones(n // 4, dtype=torch.float32, device=dev)
        self.flush_sink = torch.empty((), dtype=torch.float32, device=dev)

    def flush(self, i: int):
        """Write one buffer larger than L2, then read another, so L2 holds clean lines of
        neither the layer's inputs nor its outputs when a step starts."""
        if self.flush_mib == 0:
            return
        self.flush_w.fill_(i & 0xFF)
        self.torch.sum(self.flush_r, dim=0, out=self.flush_sink)

    def ev(self):
        return self.torch.cuda.Event(enable_timing=True)


class Workload:
    """One layer with resident inputs, its outputs, and one call captured in a CUDA graph."""

    def __init__(self, moe, cfg, dev, deterministic=False):
        import torch

        import workloads
        self.moe, self.cfg, self.dev = moe, cfg, dev
        gen_dev = dev if big_layer(cfg) else "cpu"
        self.inp = workloads.make_inputs(cfg, device=gen_dev).to(dev)
        self.layer = moe.MoELayer.from_inputs(self.inp, deterministic=deterministic)
        T, K, E, D = cfg.T, cfg.K, cfg.E, cfg.D
        self.out = torch.empty((T, D), dtype=torch.bfloat16, device=dev)
        self.idx = torch.empty((T, K), dtype=torch.int32, device=dev)
        self.tw = torch.empty((T, K), dtype=torch.float32, device=dev)
        self.counts = torch.empty((E,), dtype=torch.int32, device=dev)
        self.call()  # allocates the workspace, loads the kernels
        torch.cuda.synchronize()
        s = torch.cuda.Stream(device=dev)
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            self.call()
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        self.graph = torch.cuda.CUDAGraph()
        n0 = moe.launch_count()
        with torch.cuda.graph(self.graph):
            self.call()
        self.launches_per_call = moe.launch_count() - n0
        torch.cuda.synchronize()

    def call(self, events=None):
        self.layer(self.inp.x, out=self.out, topk_idx=self.idx, topk_w=self.tw,
                   counts=self.counts, step_events=events)

    def routing_stats(self):
        cnt = self.counts.cpu()
        return int((cnt > 0).sum()), int(cnt.max())

    def status_ok(self) -> bool:
        return self.layer.device_status() == 0


def time_graph(b: Bench, w: Workload, reps: int, flush: bool):
    """Per-replay milliseconds of the captured layer call (events around each replay)."""
    torch = b.torch
    stream = torch.cuda.current_stream()
    ea = [b.ev() for _ in range(reps)]
    eb = [b.ev() for _ in range(reps)]
    torch.cuda.synchronize()
    for i in range(reps):
        if flush:
            b.flush(i)
        ea[i].record(stream)
        w.graph.replay()
        eb[i].record(stream)
    torch.cuda.synchronize()
    return [a.elapsed_time(c) for a, c in zip(ea, eb)]


def kernel_breakdown(b: Bench, w: Workload, reps: int):
    """Milliseconds per layer step from eager calls with an event at every step boundary
    the call launches work for (events between kernels stop programmatic dependent launch,
    so this pass is slower than the graph replays), and the gate_up launch time from eager
    calls that mark only its two ends."""
    moe, torch = w.moe, b.torch
    names = moe.STEP_EVENT_NAMES
    stream = torch.cuda.current_stream()

    def run(which):
        evs = []
        for i in range(reps):
            e = [b.ev() if n in which else None for n in names]
            for x in e:
                if x is not None:
                    x.record(stream)  # creates the handle; the library re-records it
            evs.append(e)
        arrs = [moe.event_array(e) for e in evs]
        torch.cuda.synchronize()
        for i in range(reps):
            b.flush(i)
            w.call(arrs[i])
        torch.cuda.synchronize()
        return evs

    evs = run(set(names))
    steps = {n: 0.0 for n in names[1:-1]}
    for e in evs:
        for j, n in enumerate(names[1:-1], start=1):
            steps[n] += e[j].elapsed_time(e[j + 1])
    # only the steps that launch kernels of their own (moe_layer_plan): a fused step's time
    # is inside the step that runs it
    ran, _ = w.layer.plan(w.cfg.T)
    per_kernel = {n: steps[n] / reps for n in names[1:-1] if n in ran}
    step_ms = sum(e[0].elapsed_time(e[-1]) for e in evs) / reps
    ix = {n: i for i, n in enumerate(names)}
    evs = run({"start", "gate_up", "down", "end"})
    gu = [e[ix["gate_up"]].elapsed_time(e[ix["down"]]) for e in evs]
    return per_kernel, step_ms, statistics.mean(gu)


def measure(b: Bench, moe, cfg, peaks, src, reps: int, cpu_budget: float, gpu_id: str):
    """One per_config row: cold and hot medians of >= 50 graph replays, the layer
    roofline, per-kernel times, clocks, and the oracle on a bounded sample."""
    torch = b.torch
    w = Workload(moe, cfg, b.dev)
    for i in range(5):
        b.flush(i)
        w.graph.replay()
    torch.cuda.synchronize()
    sampler = ClockSampler(gpu_id)
    sampler.start()
    cold = time_graph(b, w, reps, flush=True)
    clocks = sampler.stop()
    hot = time_graph(b, w, reps, flush=False)
    if not w.status_ok():
        raise RuntimeError(f"{cfg.name}: device status is not ok")
    U, max_rows = w.routing_stats()
    per_kernel, bd_ms, gu_ms = kernel_breakdown(b, w, min(reps, 20))
    med = statistics.median(cold)
    row = {
        "workload": describe(cfg), "U": U, "max_rows_per_expert": max_rows,
        "median_ms": med, "mean_ms": statistics.mean(cold), "reps": reps,
        "hot_l2_median_ms": statistics.median(hot),
        "tokens_per_s": cfg.T / (med / 1e3),
        "layer_roofline": layer_roofline(cfg, U, med, peaks, src),
        "kernel_ms": per_kernel,
        "kernel_ms_note": f"eager calls with an event at every step boundary "
                          f"({bd_ms:.4f} ms/step there)",
        "gate_up_ms": gu_ms,
        "launches_per_call": w.launches_per_call,
        "clocks": clocks,
    }
    if cpu_budget > 0:
        row["cpu_baseline"] = cpu_baseline(w.inp, cpu_budget)
    del w
    torch.cuda.empty_cache()
    return row


def profile_calls(moe, cfg, dev, n: int, deterministic: bool) -> int:
    """n eager calls of the layer (each launches the kernels moe_layer_plan lists, in that
    order), then the plan on stdout: the launch sequence an ncu -s/-c selection counts on."""
    import torch

    import workloads
    gen_dev = dev if big_layer(cfg) else "cpu"
    inp = workloads.make_inputs(cfg, device=gen_dev).to(dev)
    layer = moe.MoELayer.from_inputs(inp, deterministic=deterministic)
    out = torch.empty((cfg.T, cfg.D), dtype=torch.bfloat16, device=dev)
    for _ in range(n):
        layer(inp.x, out=out)
    torch.cuda.synchronize()
    if layer.device_status() != 0:
        raise RuntimeError("device status is not ok")
    steps, launches = layer.plan(cfg.T)
    print(json.dumps({"workload": describe(cfg), "calls": n, "steps": steps,
                      "launches_per_call": launches}), flush=True)
    return 0


def dry_run(args, rank, world):
    """Launcher check without a GPU: every rank joins a gloo group, reports a synthetic
    per-rank time, and rank 0 prints the contract line built from the slowest rank."""
    import torch.distributed as dist
    if world > 1:
        dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    local_ms = args.steps * (1.0 + 0.5 * rank)
    slowest = max_over_ranks(local_ms)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps({"metric": METRIC, "value": whole_job_rate(world, 64, args.steps, slowest),
                          "unit": UNIT, "n_gpus": world, "steps": args.steps,
                          "warmup": args.warmup, "ms_per_step": slowest / args.steps,
                          "dry_run": True}), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default=HEADLINE)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-config", action="store_true",
                    help="time only the --config workload (the per_config rows run only at "
                         "N = 1)")
    ap.add_argument("--per-config-reps", type=int, default=50)
    ap.add_argument("--deterministic", action="store_true")
    ap.add_argument("--flush-mib", type=int, default=FLUSH_BYTES >> 20,
                    help="L2 flush buffer written before each timed step (0: none, for "
                         "profiler runs that flush caches themselves)")
    ap.add_argument("--dry-run", action="store_true",
                    help="check the multi-rank launch path on CPU (gloo), no GPU work")
    ap.add_argument("--profile-calls", type=int, default=0,
                    help="run this many eager layer calls of --config and exit, no timing "
                         "(a fixed launch sequence for an external profiler; --deterministic "
                         "applies)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.gpus < 1:
        ap.error("--gpus must be >= 1")
    os.environ.setdefault("OMP_NUM_THREADS", str(os.cpu_count() or 1))

    if "WORLD_SIZE" not in os.environ:
        if args.gpus > 1 and args.impl == "ours":
            return launch_ranks(args.gpus, sys.argv[1:])
    elif int(os.environ["WORLD_SIZE"]) != args.gpus:
        ap.error(f"--gpus {args.gpus} disagrees with WORLD_SIZE={os.environ['WORLD_SIZE']}")
    rank, world, local_rank = rank_env()
    if args.impl == "reference":
        world = max(world, args.gpus)
    if args.dry_run:
        return dry_run(args, rank, world)

    import workloads
    cfg = workloads.CONFIGS[args.config]
    if args.impl == "reference":
        return run_reference(args, cfg, world, rank)

    import torch
    import torch.distributed as dist

    import top_routing_grouped_03_b200 as moe

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    if args.profile_calls > 0:
        return profile_calls(moe, cfg, dev, args.profile_calls, args.deterministic)
    b = Bench(dev, args.flush_mib)
    w = Workload(moe, cfg, dev, deterministic=args.deterministic)
    stream = torch.cuda.current_stream()
    T = cfg.T
    for i in range(args.warmup):
        b.flush(i)
        w.graph.replay()
    torch.cuda.synchronize()
    if not w.status_ok():
        raise RuntimeError("device status after warm-up is not ok")

    ea = [b.ev() for _ in range(args.steps)]
    eb = [b.ev() for _ in range(args.steps)]
    props = torch.cuda.get_device_properties(dev)
    gpu_id = f"GPU-{props.uuid}"
    sampler = ClockSampler(gpu_id)
    sampler.start()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    for i in range(args.steps):
        b.flush(i)
        ea[i].record(stream)
        w.graph.replay()
        eb[i].record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    step_ms = [a.elapsed_time(c) for a, c in zip(ea, eb)]
    if not w.status_ok():
        raise RuntimeError("device status after the timed steps is not ok")
    total_ms = max_over_ranks(sum(step_ms), dev)
    ms_per_step = total_ms / args.steps
    value = whole_job_rate(world, T, args.steps, total_ms)
    hot_ms = statistics.median(time_graph(b, w, max(args.steps, 50), flush=False))

    # per-kernel times and the gate_up launch (eager calls, events at step boundaries)
    per_kernel, bd_step_ms, gu_ms = kernel_breakdown(b, w, args.steps)

    # ---- end to end through the public API: pinned host x in, pinned host y out, eager
    x_host = w.inp.x.cpu().pin_memory()
    y_host = torch.empty((T, cfg.D), dtype=torch.bfloat16).pin_memory()
    x_dev = torch.empty_like(w.inp.x)
    for i in range(args.warmup):
        w.layer.forward_host(x_host, y_host, x_dev, w.out)
    e_a = [b.ev() for _ in range(args.steps)]
    e_b = [b.ev() for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    for i in range(args.steps):
        b.flush(i)
        e_a[i].record(stream)
        w.layer.forward_host(x_host, y_host, x_dev, w.out)
        e_b[i].record(stream)
    torch.cuda.synchronize()
    seq_ms = max_over_ranks(sum(a.elapsed_time(c) for a, c in zip(e_a, e_b)), dev)
    # the same steps through the pipelined entry point: each step's copies in and out run
    # on copy streams while the layer runs the neighbouring steps (weights far larger than
    # L2, so no flush between steps is needed)
    y_hosts = [y_host, torch.empty_like(y_host).pin_memory()]
    x_devs = [x_dev, torch.empty_like(x_dev)]
    y_devs = [w.out, torch.empty_like(w.out)]

    def pipeline(n):
        w.layer.forward_host_stream([x_host] * n, [y_hosts[i % 2] for i in range(n)], x_devs,
                                    y_devs)

    pipeline(args.warmup)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    p_a, p_b = b.ev(), b.ev()
    p_a.record(stream)
    pipeline(args.steps)
    p_b.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(p_a.elapsed_time(p_b), dev)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    e2e = {"value": whole_job_rate(world, T, args.steps, e2e_ms), "unit": UNIT,
           "h2d_bytes_per_step": x_host.numel() * x_host.element_size(),
           "d2h_bytes_per_step": y_host.numel() * y_host.element_size(),
           "api": "MoELayer.forward_host_stream (copies of each step overlap the neighbouring "
                  "steps' layer calls)",
           "sequential": {"value": whole_job_rate(world, T, args.steps, seq_ms),
                          "api": "MoELayer.forward_host (copy in, layer, copy out in turn)"}}

    if rank != 0:
        return 0

    U, max_rows = w.routing_stats()
    peaks, src = load_peaks()
    peak_hbm = peaks["hbm_gbs"]
    peak_tc = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    gu_bytes, gu_flops = gate_up_bytes(cfg, U), gate_up_flops(cfg)
    if gu_flops / (peak_tc * 1e12) > gu_bytes / (peak_hbm * 1e9):
        roof = {"bound": "tensor", "achieved": gu_flops / (gu_ms / 1e3) / 1e12, "peak": peak_tc,
                "unit": "TFLOP/s", "peak_source": f"{src} (bf16_tflops, burst)",
                "algorithmic_flops_per_launch": gu_flops}
        roof["frac_nominal"] = roof["achieved"] / NOMINAL_PEAKS["bf16_tflops"]
    else:
        roof = {"bound": "hbm", "achieved": gu_bytes / (gu_ms / 1e3) / 1e9, "peak": peak_hbm,
                "unit": "GB/s", "peak_source": f"{src} (hbm_gbs)"}
        roof["frac_nominal"] = roof["achieved"] / NOMINAL_PEAKS["hbm_gbs"]
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = ncu_traffic("grouped_gemm_gate_up", cfg.name)
    roof["algorithmic_bytes_per_launch"] = gu_bytes
    roof["avg_launch_ms"] = gu_ms
    roof["kernel"] = "grouped_gemm gate_up + SwiGLU"
    roof["timing"] = (f"CUDA events around the gate_up launch in {args.steps} eager layer "
                      f"calls right after the timed steps (L2 flushed before each)")
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {
            "workload": describe(cfg), "global_batch": world * T, "tokens_per_gpu": T,
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
            "l2": "flushed before every timed step (512 MiB write, then 512 MiB read), "
                  "outside the timed interval",
            "timing": "one CUDA-graph replay of the layer call per step, CUDA events "
                      "around each replay",
            "routing_U": U, "max_rows_per_expert": max_rows,
            "deterministic_combine": bool(args.deterministic),
        },
        "median_ms": statistics.median(step_ms),
        "hot_l2_median_ms": hot_ms,
        "roofline": roof,
        "layer_roofline": layer_roofline(cfg, U, ms_per_step, peaks, src),
        "kernel_ms": per_kernel,
        "kernel_ms_note": f"eager calls with an event at every step boundary "
                          f"({bd_step_ms:.4f} ms/step there)",
        "e2e": e2e,
        "gpu_launches": w.launches_per_call * args.steps,
        "clocks": clocks,
    }
    cpu_inp = w.inp
    del w
    torch.cuda.empty_cache()
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(cpu_inp, 10.0)
    del cpu_inp
    torch.cuda.empty_cache()
    if world == 1 and not args.no_per_config:
        per = {}
        for name in PER_CONFIG:
            if name == cfg.name:
                continue
            per[name] = measure(b, moe, workloads.CONFIGS[name], peaks, src,
                                max(args.per_config_reps, 50),
                                0.0 if args.no_cpu_baseline else 3.0, gpu_id)
        line["per_config"] = per
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
