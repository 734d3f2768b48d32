#!/usr/bin/env python
"""Throughput of one top-k MoE SwiGLU layer forward on B200 GPUs.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl ours|reference]

One step = one whole layer call (router, permutation, gather, grouped gate_up + SwiGLU,
grouped down + weighted combine, bf16 output) over one batch of synthetic tokens already
resident in HBM.  L2 is flushed (512 MiB write) before every timed step, outside the timed
interval (the flush writes one 512 MiB buffer and reads another, so L2 starts each step
with clean lines); each step is timed with CUDA events recorded by the library on its stream,
and the per-kernel intervals come from the same events.  With N > 1 (torchrun, one
process per GPU) every rank runs an independent replica of the batch (no exchange): the
reported value is all ranks' tokens over the slowest rank's time.

``--impl reference`` times the CPU oracle (fp64, OpenMP) on this host instead.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import re
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE layer tokens/s on 1 B200 and % of roofline (HBM GB/s or bf16 TC util)"
UNIT = "tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
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
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.tmp, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.25)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.15)
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


def oracle_step(inp, tokens):
    import numpy as np

    import oracle
    r = oracle.route(inp.x, inp.w_router, inp.cfg.K, inp.logit_bias, inp.w_shared_gate)
    toks = np.asarray(tokens, np.int32)
    oracle.experts(inp.x, r["idx"], r["alpha"], inp.w_gate_up, inp.w_down, toks,
                   inp.w_shared_gate_up, inp.w_shared_down, r["shared_gate"])
    return len(toks)


def cpu_baseline(inp, budget_s=10.0):
    """The oracle as it stands on this host's cores: the whole batch (router over every
    token, expert sum for every token), repeated until ~budget_s of work."""
    import oracle
    oracle.build()
    T = inp.cfg.T
    n, t0 = 0, time.perf_counter()
    reps = 0
    while True:
        n += oracle_step(inp, range(T))
        reps += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    dt = time.perf_counter() - t0
    return {"value": n / dt, "unit": UNIT, "cores": int(os.environ.get("OMP_NUM_THREADS", "1")),
            "kind": "oracle",
            "sample": f"the full {T}-token batch (router + expert sum, fp64) x {reps}, {dt:.1f} s"}


def run_reference(args, cfg, world, rank):
    if rank != 0:
        return 0
    import workloads
    inp = workloads.make_inputs(cfg)
    import oracle
    oracle.build()
    t1 = time.perf_counter()
    oracle_step(inp, [0])
    per_tok = max(time.perf_counter() - t1, 1e-3)
    budget = 90.0  # seconds for the whole warmup + timed run
    ntok = int(max(1, min(cfg.T, budget / (args.steps + args.warmup) / per_tok)))
    toks = list(range(ntok))
    for _ in range(args.warmup):
        oracle_step(inp, toks)
    t0 = time.perf_counter()
    n = 0
    for _ in range(args.steps):
        n += oracle_step(inp, toks)
    dt = time.perf_counter() - t0
    value = n / dt
    cores = int(os.environ.get("OMP_NUM_THREADS", "1"))
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * dt / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": describe(cfg), "tokens_per_step": ntok},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"{ntok} token(s) per step: router over all {cfg.T} tokens "
                                   f"+ expert sum of the sampled tokens, fp64"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- GPU arm


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--config", default="decode")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--deterministic", action="store_true")
    ap.add_argument("--events", default="roofline", choices=["roofline", "ends", "all"],
                    help="step boundaries recorded in the timed steps: start/gate_up/down/end "
                         "(default), start/end only, or every kernel boundary")
    ap.add_argument("--flush-mib", type=int, default=FLUSH_BYTES >> 20,
                    help="L2 flush buffer written before each timed step (0: none, for "
                         "profiler runs that flush caches themselves)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    os.environ.setdefault("OMP_NUM_THREADS", str(os.cpu_count() or 1))

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

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

    big = cfg.T * cfg.D * cfg.E > (1 << 31)
    inp = workloads.make_inputs(cfg, device=dev if big else "cpu").to(dev)
    layer = moe.MoELayer.from_inputs(inp, deterministic=args.deterministic)
    T, K, E = cfg.T, cfg.K, cfg.E
    out = torch.empty((T, cfg.D), dtype=torch.bfloat16, device=dev)
    idx = torch.empty((T, K), dtype=torch.int32, device=dev)
    tw = torch.empty((T, K), dtype=torch.float32, device=dev)
    counts = torch.empty((E,), dtype=torch.int32, device=dev)
    # L2 flush between timed steps: write one buffer larger than L2, then read another,
    # so L2 holds clean lines when a step starts (the write-back of the dirty lines the
    # write leaves happens during the read, outside the timed interval)
    nflush = max(args.flush_mib, 1) << 20
    flush_w = torch.empty(nflush, dtype=torch.uint8, device=dev)
    flush_r = torch.ones(nflush // 4, dtype=torch.float32, device=dev)
    flush_sink = torch.empty((), dtype=torch.float32, device=dev)

    class _Flush:
        def fill_(self, v):
            if args.flush_mib == 0:
                return
            flush_w.fill_(v)
            torch.sum(flush_r, dim=0, out=flush_sink)

    flush = _Flush()
    stream = torch.cuda.current_stream()

    names = moe.STEP_EVENT_NAMES
    recorded = {"roofline": {"start", "gate_up", "down", "end"}, "ends": {"start", "end"},
                "all": set(names)}[args.events]

    def events(which):
        evs = [torch.cuda.Event(enable_timing=True) if n in which else None for n in names]
        for e in evs:
            if e is not None:
                e.record(stream)  # creates the handle; the library re-records it
        return evs

    for i in range(args.warmup):
        flush.fill_(i & 0xFF)
        layer(inp.x, out=out, topk_idx=idx, topk_w=tw, counts=counts)
    torch.cuda.synchronize()
    if layer.device_status() != 0:
        raise RuntimeError("device status after warm-up is not ok")

    step_evs = [events(recorded) for _ in range(args.steps)]
    arrs = [moe.event_array(e) for e in step_evs]
    torch.cuda.synchronize()
    props = torch.cuda.get_device_properties(dev)
    sampler = ClockSampler(f"GPU-{props.uuid}")
    sampler.start()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    n0 = moe.launch_count()
    for i in range(args.steps):
        flush.fill_(i & 0xFF)
        layer(inp.x, out=out, topk_idx=idx, topk_w=tw, counts=counts, step_events=arrs[i])
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    launches = moe.launch_count() - n0
    clocks = sampler.stop()
    if layer.device_status() != 0:
        raise RuntimeError("device status after the timed steps is not ok")

    ix = {n: i for i, n in enumerate(names)}
    total_ms = sum(evs[0].elapsed_time(evs[-1]) for evs in step_evs)
    gu_total = (sum(e[ix["gate_up"]].elapsed_time(e[ix["down"]]) for e in step_evs)
                if "gate_up" in recorded else None)

    # per-kernel breakdown: a separate pass with every boundary recorded (those marks keep
    # each kernel from overlapping its predecessor, so the pass is slower than the step)
    n_bd = min(args.steps, 100)
    bd_evs = [events(set(names)) for _ in range(n_bd)]
    bd_arrs = [moe.event_array(e) for e in bd_evs]
    torch.cuda.synchronize()
    for i in range(n_bd):
        flush.fill_(i & 0xFF)
        layer(inp.x, out=out, topk_idx=idx, topk_w=tw, counts=counts, step_events=bd_arrs[i])
    torch.cuda.synchronize()
    per_kernel = {n: 0.0 for n in names[1:-1]}
    for evs in bd_evs:
        for j, n in enumerate(names[1:-1], start=1):
            per_kernel[n] += evs[j].elapsed_time(evs[j + 1])
    bd_step_ms = sum(e[0].elapsed_time(e[-1]) for e in bd_evs) / n_bd
    if gu_total is None:
        gu_total = per_kernel["gate_up"] * args.steps / n_bd
    total_ms = max_over_ranks(total_ms, dev)
    ms_per_step = total_ms / args.steps
    value = whole_job_rate(world, T, args.steps, total_ms)

    # ---- end to end through the public API: pinned host x in, pinned host y out
    x_host = inp.x.cpu().pin_memory()
    y_host = torch.empty((T, cfg.D), dtype=torch.bfloat16).pin_memory()
    x_dev = torch.empty_like(inp.x)
    for i in range(args.warmup):
        layer.forward_host(x_host, y_host, x_dev, out)
    e_a = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    e_b = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    for i in range(args.steps):
        flush.fill_(i & 0xFF)
        e_a[i].record(stream)
        layer.forward_host(x_host, y_host, x_dev, out)
        e_b[i].record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in zip(e_a, e_b)), dev)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    e2e = {"value": whole_job_rate(world, T, args.steps, e2e_ms), "unit": UNIT,
           "h2d_bytes_per_step": x_host.numel() * x_host.element_size(),
           "d2h_bytes_per_step": y_host.numel() * y_host.element_size()}

    if rank != 0:
        return 0

    cnt = counts.cpu()
    U = int((cnt > 0).sum())
    peaks, peak_src = load_peaks()
    # tensor peak: the sustained figure (a kernel inside a long, power-capped step), the
    # burst one only when no sustained measurement exists
    tc_key = "bf16_tflops_sustained" if "bf16_tflops_sustained" in peaks else "bf16_tflops"
    peak_tc, peak_hbm = peaks[tc_key], peaks["hbm_gbs"]
    gu_ms = gu_total / args.steps
    gu_bytes = gate_up_bytes(cfg, U)
    gu_flops = gate_up_flops(cfg)
    tensor_bound = gu_flops / (peak_tc * 1e12) > gu_bytes / (peak_hbm * 1e9)
    if tensor_bound:
        roof = {"bound": "tensor", "achieved": gu_flops / (gu_ms / 1e3) / 1e12, "peak": peak_tc,
                "unit": "TFLOP/s", "peak_source": f"{peak_src} ({tc_key})",
                "algorithmic_flops_per_launch": gu_flops}
    else:
        roof = {"bound": "hbm", "achieved": gu_bytes / (gu_ms / 1e3) / 1e9, "peak": peak_hbm,
                "unit": "GB/s", "peak_source": f"{peak_src} (hbm_gbs)"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = ncu_traffic("grouped_gemm_gate_up", cfg.name)
    roof["algorithmic_bytes_per_launch"] = gu_bytes
    roof["avg_launch_ms"] = gu_ms
    roof["kernel"] = "grouped_gemm gate_up + SwiGLU"
    F, B = layer_flops(cfg), layer_bytes(cfg, U)
    t_roof = max(F / (peak_tc * 1e12), B / (peak_hbm * 1e9))
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {
            "workload": describe(cfg), "global_batch": world * T, "tokens_per_gpu": T,
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
            "l2": "flushed before every timed step (512 MiB write, then 512 MiB read), "
                  "outside the timed interval; expert weights read per step exceed L2",
            "routing_U": U, "max_rows_per_expert": int(cnt.max()),
            "deterministic_combine": bool(args.deterministic),
        },
        "roofline": roof,
        "layer_roofline": {
            "bound": "tensor" if F / (peak_tc * 1e12) > B / (peak_hbm * 1e9) else "hbm",
            "peaks": f"{peak_tc} TFLOP/s ({tc_key}), {peak_hbm} GB/s (hbm_gbs), {peak_src}",
            "flops": F, "bytes": B, "t_roof_ms": 1e3 * t_roof,
            "frac": 1e3 * t_roof / ms_per_step,
            "achieved_tflops": F / (ms_per_step / 1e3) / 1e12,
            "achieved_gbs": B / (ms_per_step / 1e3) / 1e9,
        },
        "kernel_ms": {n: v / n_bd for n, v in per_kernel.items()},
        "kernel_ms_note": f"separate {n_bd}-step pass with every kernel boundary recorded "
                          f"({bd_step_ms:.4f} ms/step there); timed steps recorded "
                          f"{sorted(recorded)}",
        "e2e": e2e,
        "gpu_launches": launches,
        "clocks": clocks,
    }
    if world == 1 and not args.no_cpu_baseline:
        cpu_inp = inp.to("cpu")
        line["cpu_baseline"] = cpu_baseline(cpu_inp)
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
