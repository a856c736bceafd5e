"""Benchmark of the fused, chunked top-K forward-KL loss (forward + backward).

    python bench.py [--gpus N --steps K --warmup W] [--impl ours|reference]
                    [--workload bf16_32k] [--chunk C]

One step = one ckl_fwd_bwd call over one batch of the workload: loss, dH and dW
for T tokens (the 32K-token case by default: T=32768, d=2880, V=201088, K=100,
chunk 2048). Inputs are seeded synthetic draws (chunked_kl_loss_logits_b200/
workloads.py), resident in HBM before the timed region; W alone (1.16 GB) is
larger than the 126 MB L2, so no flush is needed between steps. The timed
region is bracketed by a barrier and a device synchronise, timed with CUDA
events, and the max over ranks is taken. With N GPUs every rank runs its own
replica on its own batch (tokens are independent; no collective on the data
path), so scaling is weak and `value` is the tokens/s of all ranks together.

`--impl reference` times the fp64 CPU oracle on the host cores on a bounded
sample of the same workload (the oracle is the reference of this build; it is
a deliberately slow, obviously correct program, not a tuned baseline).
Prints one JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import ctypes
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "fwd+bwd tokens/s & TFLOP/s (% bf16 tensor peak) at T=32K, V=201088, K=100"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


class ClockSampler:
    """nvidia-smi samples (every 200 ms) of this GPU's SM clock and throttle reasons."""

    FIELDS = ("pci.bus_id,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, bus_id: str):
        self.bus_id = bus_id.lower()
        self.lines = []
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.t = threading.Thread(target=self._read, daemon=True)
        self.t.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.t.join(timeout=5)
        sm, smax, power, reasons = [], [], [], set()
        for ln in self.lines:
            c = [x.strip() for x in ln.split(",")]
            if len(c) < 9 or c[0].lower() != self.bus_id:
                continue
            try:
                sm.append(float(c[1]))
                smax.append(float(c[2]))
                power.append(float(c[3]))
            except ValueError:
                continue
            for name, v in zip(self.NAMES, c[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "power_w_max": max(power) if power else None,
                "power_w_median": statistics.median(power) if power else None,
                "samples": len(sm), "reasons": sorted(reasons)}


TRAFFIC_FILE = os.path.join(ROOT, "profiles", "dram_traffic_bf16_32k.md")
# The sources of the tensor-core kernels whose DRAM traffic the summary records.
KERNEL_SOURCES = ("chunked_kl_loss_logits_b200/csrc/k_tc.cu", "chunked_kl_loss_logits_b200/csrc/common.cuh",
                  "chunked_kl_loss_logits_b200/csrc/k_tc.h")


def code_text(src: str) -> str:
    """C++/CUDA source without its comments and with whitespace runs collapsed: the
    text that decides what the compiler builds (string literals hold no comment
    markers in these files)."""
    import re
    src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
    src = re.sub(r"//[^\n]*", " ", src)
    return " ".join(src.split())


def kernel_source_hash(root: str = ROOT) -> str:
    """Hash of the tensor-core kernels' code (comments and layout excluded)."""
    import hashlib
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(root, rel), encoding="utf-8") as f:
            h.update(code_text(f.read()).encode())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, workload: str, chunk: int):
    """DRAM bytes per launch of `kernel` from the committed ncu summary, or None.

    The summary records a hash of the kernel sources it was measured on; a
    changed kernel (or another workload) gives None.
    """
    import re
    if not os.path.exists(TRAFFIC_FILE):
        return None
    with open(TRAFFIC_FILE) as f:
        text = f.read()
    m = re.search(r"<!-- traffic (.*?) -->", text)
    if not m:
        return None
    kv = dict(x.split("=", 1) for x in m.group(1).split())
    if kv.get("source") != kernel_source_hash() or kv.get("workload") != workload or \
            int(kv.get("chunk", -1)) != chunk:
        return None
    val = kv.get(kernel)
    return float(val) if val is not None else None


class EnergyCounter:
    """The GPU's cumulative energy counter (NVML, millijoules since the driver loaded).

    Read-only: read() returns joules, or None where NVML or the counter is missing.
    """

    def __init__(self, bus_id: str):
        self.h = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByPciBusId(bus_id.upper())
            self.read()
        except Exception:
            self.h = None

    def read(self):
        if self.h is None:
            return None
        try:
            return self.nv.nvmlDeviceGetTotalEnergyConsumption(self.h) / 1e3
        except Exception:
            return None


def max_over_ranks(ms: float, world: int, device="cpu") -> float:
    """The slowest rank's time: every rank takes part, every rank gets the max."""
    if world == 1:
        return float(ms)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(tokens_per_rank: int, world: int, steps: int, ms_max: float) -> float:
    """Weak scaling: every rank processes its own batch; the job rate uses the slowest rank."""
    return tokens_per_rank * world * steps / (ms_max / 1e3)


def bus_id_of(dev: int) -> str:
    import torch
    p = torch.cuda.get_device_properties(dev)
    return f"{p.pci_domain_id:08x}:{p.pci_bus_id:02x}:{p.pci_device_id:02x}.0"


# Row counts of the two oracle calls each CPU-baseline step times (same in both legs).
ORACLE_ROWS = (64, 192)


def oracle_rate(x, w, steps: int = 1, warmup: int = 1):
    """Per-token rate of the fp64 oracle on the host cores, from the slope of two calls.

    W is widened to float64 once, before any timed call, so that no call pays the
    multi-GB conversion (the oracle then uses the array as it is). Every step times
    `oracle.sampled_rows` (lse, l_t, dH row and dW share of each sampled token) on
    ORACLE_ROWS[0] and on ORACLE_ROWS[1] consecutive tokens of the workload; the
    difference of the two times over the difference of the row counts is the
    oracle's time per token, free of the per-call fixed costs (passes over W, the
    V x d dW allocation). Returns (tokens/s of each timed step, per-call fixed
    seconds of each step, row counts, cores).
    """
    import oracle
    import threadpoolctl
    info = threadpoolctl.threadpool_info()
    cores = max([i.get("num_threads", 1) for i in info] + [1])
    W64 = np.asarray(x["W"], dtype=np.float64)  # untimed, once
    n_a, n_b = ORACLE_ROWS
    # one untimed call first: starting the BLAS threads and touching fresh pages are
    # not per-token costs, whatever the warm-up count
    oracle.sampled_rows(x["H"], W64, x["idx"], x["logit"], np.arange(min(n_a, w.T)), x["mask"],
                        with_dW=True)
    rates, fixed = [], []
    for s in range(warmup + steps):
        t_call = []
        for n in (n_a, n_b):
            start = (s * n_b) % max(1, w.T - n_b)
            rows = np.arange(start, start + n)
            t0 = time.perf_counter()
            oracle.sampled_rows(x["H"], W64, x["idx"], x["logit"], rows, x["mask"], with_dW=True)
            t_call.append(time.perf_counter() - t0)
        if t_call[1] > t_call[0]:
            per_tok = (t_call[1] - t_call[0]) / (n_b - n_a)
            fix = t_call[0] - n_a * per_tok
        else:
            # the fixed cost swamps the per-token one (a small vocabulary) and the two
            # times do not order: the larger call's whole time per token, a lower rate
            per_tok = t_call[1] / n_b
            fix = float("nan")
        if s >= warmup:
            rates.append(1.0 / per_tok)
            fixed.append(fix)
    return rates, fixed, (n_a, n_b), cores


def oracle_sample_text(rows, steps, fixed):
    slopes = [f for f in fixed if f == f]  # NaN marks a step timed by its whole call
    text = (f"slope of two oracle calls per step ({rows[0]} and {rows[1]} consecutive tokens of the "
            f"workload; full per-token path: lse, l_t, dH row, dW share; fp64 numpy/BLAS, W widened "
            f"to fp64 once before timing), {steps} timed step(s)")
    if slopes:
        text += f"; per-call fixed cost {statistics.median(slopes):.2f} s excluded"
    if len(slopes) < len(fixed):
        text += (f"; {len(fixed) - len(slopes)} step(s) whose two times did not order timed by the "
                 f"{rows[1]}-token call's whole time, fixed cost included")
    return text


def bench_config(w, mask, chunk, recompute, world):
    """The workload description of the bench line (the same for both arms)."""
    return {"workload": w.name, "T": w.T, "d": w.d, "V": w.V, "K": w.K, "chunk": chunk,
            "valid_tokens": int(w.T if mask is None else int(mask.astype(bool).sum())),
            "backward": ("recompute logits" if recompute or w.dtype != "bf16"
                         else "stored exp(z), bf16"),
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
            "l2": "no flush: inputs larger than L2 (W alone is 1.16 GB)"}


def run_reference(args, w, rank, world):
    if rank != 0:
        return
    from chunked_kl_loss_logits_b200.workloads import make_inputs
    x = make_inputs(w)
    rates, fixed, rows, cores = oracle_rate(x, w, steps=args.steps, warmup=args.warmup)
    value = float(len(rates) / sum(1.0 / r for r in rates))  # tokens/s over the timed steps
    ms = 1000.0 * (rows[1] - rows[0]) / value
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": bench_config(w, x["mask"], args.chunk or w.chunk, args.recompute, world),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": oracle_sample_text(rows, args.steps, fixed)},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_ours(args, w, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    from chunked_kl_loss_logits_b200 import ckl
    from chunked_kl_loss_logits_b200.workloads import make_inputs

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    chunk = args.chunk or w.chunk
    x = make_inputs(w, seed=w.seed + 7919 * rank)
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    H = torch.from_numpy(x["H"]).to(dev).to(tdt)
    W = torch.from_numpy(x["W"]).to(dev).to(tdt)
    idx = torch.from_numpy(x["idx"]).to(dev)
    logit = torch.from_numpy(x["logit"]).to(dev)
    mask = None if x["mask"] is None else torch.from_numpy(x["mask"]).to(dev)
    h = ckl.ChunkedKL(w.V, w.d, w.K, dtype=tdt, max_chunk=chunk, device=dev)
    if w.dtype == "bf16":
        h.set_recompute(args.recompute)
    ws = h.workspace(w.T, chunk)
    out = (torch.empty((), dtype=torch.float32, device=dev), torch.empty_like(H),
           torch.empty((w.V, w.d), dtype=torch.float32, device=dev))
    stream = torch.cuda.current_stream(dev)
    torch.cuda.reset_peak_memory_stats(dev)

    def step():
        h.fwd_bwd(H, W, idx, logit, mask, chunk=chunk, out=out, workspace=ws, sync=False)

    for _ in range(args.warmup):
        step()
    h.sync_status()

    def barrier():
        if world > 1:
            dist.barrier()

    sampler = ClockSampler(bus_id_of(local_rank))
    energy = EnergyCounter(bus_id_of(local_rank))
    h.profile_enable(True, 64 + args.steps * (12 * ((w.T + chunk - 1) // chunk) + 8))
    n_launch0 = h.launch_count()
    barrier()
    torch.cuda.synchronize(dev)
    sampler.start()
    j0 = energy.read()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    # one event between consecutive steps as well (recorded on the stream, no sync)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(max(0, args.steps - 1))]
    e0.record(stream)
    for i in range(args.steps):
        step()
        if i < args.steps - 1:
            ev[i].record(stream)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    j1 = energy.read()
    barrier()
    clocks = sampler.stop()
    launches = h.launch_count() - n_launch0
    h.sync_status()
    ms_max = max_over_ranks(e0.elapsed_time(e1), world, dev)
    marks = [e0] + ev + [e1]
    per_step = [a.elapsed_time(b) for a, b in zip(marks, marks[1:])]
    stats = h.profile_collect()
    h.profile_enable(False, 0)
    peak_mem = torch.cuda.max_memory_allocated(dev) / 2**30
    if not clocks.get("samples") and sampler.proc is not None:
        # the timed region was shorter than the 200 ms sampling period: sample over
        # an untimed continuation of the same step (about half a second), and say so
        extra = ClockSampler(bus_id_of(local_rank))
        extra.start()
        t_end = time.time() + 0.6
        while time.time() < t_end:
            step()
            torch.cuda.synchronize(dev)
        clocks = extra.stop()
        clocks["sampled"] = "untimed continuation of the same step (timed region < 200 ms)"

    # end to end: per-step inputs from pinned host memory, loss read back, every step
    Hh = H.cpu().pin_memory()
    ih = idx.cpu().pin_memory()
    lh = logit.cpu().pin_memory()
    mh = None if mask is None else mask.cpu().pin_memory()
    stag = (torch.empty_like(H), torch.empty_like(idx), torch.empty_like(logit),
            None if mask is None else torch.empty_like(mask))
    h2d = Hh.numel() * Hh.element_size() + ih.numel() * 4 + lh.numel() * 4 + \
        (0 if mh is None else mh.numel())
    h.fwd_bwd_from_host(Hh, ih, lh, mh, stag, W, chunk, out, ws)
    barrier()
    torch.cuda.synchronize(dev)
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    for _ in range(args.steps):
        h.fwd_bwd_from_host(Hh, ih, lh, mh, stag, W, chunk, out, ws)
    f1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    e2e_ms = max_over_ranks(f0.elapsed_time(f1), world, dev)

    # the pages' two other loss forms beside this library, on this step's inputs
    # (rank 0 at N = 1; the library's own buffers are released first)
    compare = None
    if rank == 0 and world == 1 and not args.no_compare and w.dtype == "bf16" and mask is None:
        del out, ws, stag, Hh, ih, lh, mh
        h.close()
        torch.cuda.synchronize(dev)
        torch.cuda.empty_cache()
        free, _ = torch.cuda.mem_get_info(dev)
        compare = [{k: v for k, v in r.items() if k not in ("kind", "workload", "V", "d", "K")}
                   for r in compare_forms(w, w.T, H, W, idx, logit, chunk, 2, dev, 0.92 * free)]

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rates, fixed, rows, cores = oracle_rate(x, w, steps=2, warmup=1)
        cpu = {"value": float(len(rates) / sum(1.0 / r for r in rates)), "unit": "tokens/s",
               "cores": cores, "kind": "oracle",
               "sample": oracle_sample_text(rows, len(rates), fixed)}
    if rank != 0:
        return

    peaks, peak_src = load_peaks()
    value = job_tokens_per_s(w.T, world, args.steps, ms_max)
    step_ms = ms_max / args.steps
    useful = 6.0 * w.T * w.V * w.d
    recompute = args.recompute or w.dtype != "bf16"
    executed = (8.0 if recompute else 6.0) * w.T * w.V * w.d  # stored mode forms the logits once
    pk_sus = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    pk_burst = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    kern = sorted(stats, key=lambda s: -s["total_ms"])
    total_k = sum(s["total_ms"] for s in kern) or 1.0
    top = kern[0]
    avg_ms = top["total_ms"] / top["launches"]
    if top["flops"] > 0:
        achieved = top["flops"] / top["launches"] / (avg_ms / 1e3) / 1e12
        roof = {"kernel": top["name"], "bound": "tensor", "achieved": achieved, "peak": pk_sus,
                "unit": "TFLOP/s", "frac": achieved / pk_sus,
                "traffic": recorded_traffic(top["name"], w.name, chunk),
                "peak_source": f"{peak_src} bf16_tflops_sustained (kernel timed inside a long step)",
                "flops_per_launch": top["flops"] / top["launches"], "avg_launch_ms": avg_ms}
    else:
        achieved = top["bytes"] / top["launches"] / (avg_ms / 1e3) / 1e9
        hbm = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
        roof = {"kernel": top["name"], "bound": "hbm", "achieved": achieved, "peak": hbm,
                "unit": "GB/s", "frac": achieved / hbm,
                "traffic": recorded_traffic(top["name"], w.name, chunk),
                "peak_source": f"{peak_src} hbm_gbs", "avg_launch_ms": avg_ms}
    if j0 is not None and j1 is not None:
        # the board's energy counter over the timed region (rank 0's GPU): joules per step
        clocks["joules_per_step"] = (j1 - j0) / args.steps
        clocks["joules_source"] = "NVML total energy counter over the timed region"
    elif clocks.get("power_w_median"):
        # board power under load x step time: the energy one step costs (the cap binds)
        clocks["joules_per_step"] = clocks["power_w_median"] * step_ms / 1e3
        clocks["joules_source"] = "median sampled board power x step time"
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_ms,
        "ms_per_step_median_rank0": statistics.median(per_step),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if w.dtype == "bf16" else "f32",
        "data": "synthetic",
        "config": bench_config(w, x["mask"], chunk, args.recompute, world),
        "tflops_useful": useful / (step_ms / 1e3) / 1e12,
        "tflops_executed": executed / (step_ms / 1e3) / 1e12,
        "frac_peak_useful": useful / (step_ms / 1e3) / 1e12 / pk_burst,
        "frac_peak_executed": executed / (step_ms / 1e3) / 1e12 / pk_burst,
        "peak_tflops_used": {"value": pk_burst, "source": f"{peak_src} bf16_tflops"},
        "peak_mem_gib": peak_mem,
        "roofline": roof,
        "cpu_baseline": cpu,
        "e2e": {"value": job_tokens_per_s(w.T, world, args.steps, e2e_ms), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": 4},
        "gpu_launches": launches,
        "compare": compare,
        "clocks": clocks,
        "kernels": [{"name": s["name"], "launches": s["launches"],
                     "ms_per_step": s["total_ms"] / args.steps,
                     "share": s["total_ms"] / total_k,
                     **({"tflops": s["flops"] / (s["total_ms"] / 1e3) / 1e12} if s["flops"] else {}),
                     **({"gbs": s["bytes"] / (s["total_ms"] / 1e3) / 1e9}
                        if s["bytes"] and not s["flops"] else {})}
                    for s in kern],
    }
    print(json.dumps(line), flush=True)


def run_sweep(args, w):
    """256K-token workload: throughput vs chunk, and peak device memory vs T.

    Prints one JSON line per point (kind "chunk_sweep" or "memory_sweep"). Peak
    memory counts everything the step allocates through torch: inputs, outputs
    and the library's workspace.
    """
    import torch

    from chunked_kl_loss_logits_b200 import ckl
    from chunked_kl_loss_logits_b200.workloads import WORKLOADS, make_inputs
    w = WORKLOADS["bf16_256k"]
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    x = make_inputs(w)
    H_all = torch.from_numpy(x["H"]).to(dev).to(torch.bfloat16)
    W = torch.from_numpy(x["W"]).to(dev).to(torch.bfloat16)
    idx_all = torch.from_numpy(x["idx"]).to(dev)
    lg_all = torch.from_numpy(x["logit"]).to(dev)
    del x
    stream = torch.cuda.current_stream(dev)
    for chunk in w.chunk_sweep:
        h = ckl.ChunkedKL(w.V, w.d, w.K, max_chunk=chunk, device=dev)
        ws = h.workspace(w.T, chunk)
        out = (torch.empty((), device=dev), torch.empty_like(H_all),
               torch.empty((w.V, w.d), dtype=torch.float32, device=dev))
        for _ in range(2):
            h.fwd_bwd(H_all, W, idx_all, lg_all, None, chunk=chunk, out=out, workspace=ws, sync=False)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n_chunks = (w.T + chunk - 1) // chunk
        h.profile_enable(True, args.sweep_steps * (10 * n_chunks + 8))
        torch.cuda.synchronize(dev)
        e0.record(stream)
        for _ in range(args.sweep_steps):
            h.fwd_bwd(H_all, W, idx_all, lg_all, None, chunk=chunk, out=out, workspace=ws, sync=False)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        h.sync_status()
        ms = e0.elapsed_time(e1) / args.sweep_steps
        kern = {k["name"]: round(k["total_ms"] / args.sweep_steps, 2) for k in h.profile_collect()}
        print(json.dumps({"kind": "chunk_sweep", "workload": w.name, "T": w.T, "chunk": chunk,
                          "ms_per_step": ms, "tokens_per_s": w.T / (ms / 1e3),
                          "tflops_useful": 6.0 * w.T * w.V * w.d / (ms / 1e3) / 1e12,
                          "workspace_gib": ws.numel() / 2**30, "kernel_ms_per_step": kern}),
              flush=True)
        del out, ws
        h.close()
    chunk = 4096
    for T in (4096, 8192, 16384, 32768, 65536, 131072, 262144):
        torch.cuda.synchronize(dev)
        torch.cuda.empty_cache()
        H = H_all[:T].clone()
        idx = idx_all[:T].clone()
        lg = lg_all[:T].clone()
        torch.cuda.reset_peak_memory_stats(dev)
        base = torch.cuda.memory_allocated(dev)
        h = ckl.ChunkedKL(w.V, w.d, w.K, max_chunk=chunk, device=dev)
        loss, dH, dW = h.fwd_bwd(H, W, idx, lg, None, chunk=chunk)
        torch.cuda.synchronize(dev)
        peak = torch.cuda.max_memory_allocated(dev)
        print(json.dumps({"kind": "memory_sweep", "workload": w.name, "T": T, "chunk": chunk,
                          "peak_gib_step": (peak - base) / 2**30,
                          "peak_gib_with_inputs": (peak - base + (H.numel() * 2 + idx.numel() * 8)) / 2**30,
                          "resident_W_gib": W.numel() * 2 / 2**30}), flush=True)
        del loss, dH, dW, H, idx, lg
        h.close()


def _dense_kl(H, W, idx, logit):
    """Full Dense KL in plain PyTorch: the cached top-K probabilities scattered into
    a T x V teacher, compared with the student's dense log-softmax (autograd)."""
    import torch
    z = H @ W.t()
    logq = torch.log_softmax(z.float(), dim=-1)
    P = torch.zeros_like(logq).scatter_add_(1, idx.long(), torch.softmax(logit.float(), dim=-1))
    return torch.nn.functional.kl_div(logq, P, reduction="sum") / H.shape[0]


def _forward_chunked_kl(H, W, idx, logit, chunk):
    """Forward-Chunked Loss in plain PyTorch: sparse teacher, the loss evaluated in
    sequence chunks, but the full student logits come from one projection and
    autograd keeps them for the backward."""
    import torch
    z = H @ W.t()
    total = z.new_zeros((), dtype=torch.float32)
    for t0 in range(0, H.shape[0], chunk):
        zc = z[t0:t0 + chunk].float()
        lp = torch.log_softmax(logit[t0:t0 + chunk], dim=-1)
        p = lp.exp()
        lse = torch.logsumexp(zc, dim=-1)
        zk = zc.gather(1, idx[t0:t0 + chunk].long())
        total = total + (p * lp).sum() - (p * zk).sum() + lse.sum()
    return total / H.shape[0]


def compare_forms(w, T, H0, W0, idx, lg, chunk, steps, dev, budget):
    """One sequence length: the pages' two other loss forms and this library on the same inputs.

    Returns one record per method: peak device memory above the inputs and mean
    forward + backward time over `steps` steps (CUDA events, after one untimed
    step). A form whose estimated footprint exceeds `budget` bytes is not run
    (reported as skipped); an out-of-memory exception is reported, not raised.
    """
    import torch

    from chunked_kl_loss_logits_b200 import ckl
    # bytes per T x V element held at the peak, as measured at 4K-32K tokens
    # (dense: bf16 z and its grad plus ~4 fp32 T x V tensors; forward-chunked: bf16 z,
    # its grad and one fp32 chunk copy), with a margin
    est = {"dense_kl": T * w.V * 23, "forward_chunked": T * w.V * 8.5, "ckl": 0}
    recs = []
    for method in ("dense_kl", "forward_chunked", "ckl"):
        rec = {"kind": "compare", "method": method, "workload": w.name, "T": T, "V": w.V,
               "d": w.d, "K": w.K, "chunk": chunk if method != "dense_kl" else None}
        if est[method] > budget:
            rec["status"] = "skipped: estimated %.0f GiB above the %.0f GiB budget" % (
                est[method] / 2**30, budget / 2**30)
            recs.append(rec)
            continue
        H = H0.detach().clone().requires_grad_(method != "ckl")
        W = W0.detach().clone().requires_grad_(method != "ckl")
        h = ckl.ChunkedKL(w.V, w.d, w.K, max_chunk=chunk, device=dev) if method == "ckl" else None

        def step():
            if method == "ckl":
                return h.fwd_bwd(H, W, idx, lg, None, chunk=chunk, sync=False)[0]
            H.grad = W.grad = None
            loss = _dense_kl(H, W, idx, lg) if method == "dense_kl" else \
                _forward_chunked_kl(H, W, idx, lg, chunk)
            loss.backward()
            return loss.detach()

        try:
            torch.cuda.synchronize(dev)
            torch.cuda.empty_cache()
            base = torch.cuda.memory_allocated(dev)
            torch.cuda.reset_peak_memory_stats(dev)
            loss = step()
            torch.cuda.synchronize(dev)
            peak = torch.cuda.max_memory_allocated(dev) - base
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(steps):
                loss = step()
            e1.record()
            torch.cuda.synchronize(dev)
            ms = e0.elapsed_time(e1) / steps
            rec.update(status="ok", loss=float(loss), peak_gib_above_inputs=peak / 2**30,
                       ms_per_step=ms, tokens_per_s=T / (ms / 1e3),
                       tflops_useful=6.0 * T * w.V * w.d / (ms / 1e3) / 1e12)
        except torch.cuda.OutOfMemoryError as e:
            rec["status"] = "out of memory: " + str(e).splitlines()[0][:120]
        recs.append(rec)
        del H, W
        if h is not None:
            h.close()
        torch.cuda.synchronize(dev)
        torch.cuda.empty_cache()
    return recs


def run_compare(args, w):
    """The pages' two other loss forms, in plain PyTorch on this GPU, beside this library.

    For T in a range of sequence lengths on the workload's (V, d, K): peak device
    memory above the inputs and mean forward + backward time of each form, one JSON
    line per (method, T). Inputs are the workload's own (distinct teacher ids, so
    the dense scatter and the sparse forms agree).
    """
    import torch

    from chunked_kl_loss_logits_b200.workloads import make_inputs
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    chunk = args.chunk or w.chunk
    free, total = torch.cuda.mem_get_info(dev)
    budget = 0.8 * free
    for T in args.compare_tokens:
        x = make_inputs(w, T=T)
        H0 = torch.from_numpy(x["H"]).to(dev).to(torch.bfloat16)
        W0 = torch.from_numpy(x["W"]).to(dev).to(torch.bfloat16)
        idx = torch.from_numpy(x["idx"]).to(dev)
        lg = torch.from_numpy(x["logit"]).to(dev)
        del x
        for rec in compare_forms(w, T, H0, W0, idx, lg, chunk, args.compare_steps, dev, budget):
            print(json.dumps(rec), flush=True)
        del H0, W0, idx, lg


def run_graph_compare(args, w):
    """One workload's step, eager vs captured once in a CUDA graph and replayed.

    Prints one JSON line (kind "graph"): mean ms per step of each over the same
    number of timed steps (CUDA events, after warm-up). The graph holds the
    call's launches, memsets and copies; replaying it removes the host launch
    cost, which matters when the kernels are short (small workloads).
    """
    import torch

    from chunked_kl_loss_logits_b200 import ckl
    from chunked_kl_loss_logits_b200.workloads import make_inputs
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    chunk = args.chunk or w.chunk
    x = make_inputs(w)
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    H = torch.from_numpy(x["H"]).to(dev).to(tdt)
    W = torch.from_numpy(x["W"]).to(dev).to(tdt)
    idx = torch.from_numpy(x["idx"]).to(dev)
    logit = torch.from_numpy(x["logit"]).to(dev)
    mask = None if x["mask"] is None else torch.from_numpy(x["mask"]).to(dev)
    h = ckl.ChunkedKL(w.V, w.d, w.K, dtype=tdt, max_chunk=chunk, device=dev)
    ws = h.workspace(w.T, chunk)
    out = (torch.empty((), dtype=torch.float32, device=dev), torch.empty_like(H),
           torch.empty((w.V, w.d), dtype=torch.float32, device=dev))

    def step():
        h.fwd_bwd(H, W, idx, logit, mask, chunk=chunk, out=out, workspace=ws, sync=False)

    side = torch.cuda.Stream(dev)
    side.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(side):
        for _ in range(max(3, args.warmup)):
            step()
    torch.cuda.current_stream(dev).wait_stream(side)
    torch.cuda.synchronize(dev)
    n0 = h.launch_count()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    per_step = h.launch_count() - n0
    h.sync_status()

    def timed(fn):
        for _ in range(max(3, args.warmup)):
            fn()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(args.steps):
            fn()
        e1.record()
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1) / args.steps

    eager = timed(step)
    graph = timed(g.replay)
    h.sync_status()
    print(json.dumps({"kind": "graph", "workload": w.name, "T": w.T, "chunk": chunk,
                      "steps": args.steps, "launches_per_step": per_step,
                      "eager_ms": eager, "graph_ms": graph,
                      "tokens_per_s_eager": w.T / (eager / 1e3),
                      "tokens_per_s_graph": w.T / (graph / 1e3)}), flush=True)
    del g
    h.close()


def run_topk_cache(args, w):
    """Teacher top-K cache builder on one workload's shape: tokens/s of one cache pass.

    The teacher here has the student's shape (same V and d); its hidden states
    are the workload's H. Prints one JSON line (kind "topk_cache"). The builder
    forms every logit twice (a max pass and an emit pass), so it executes 4TVd
    flops for the 2TVd of one logit contraction.
    """
    import torch

    from chunked_kl_loss_logits_b200 import ckl
    from chunked_kl_loss_logits_b200.workloads import make_inputs
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    x = make_inputs(w)
    H = torch.from_numpy(x["H"]).to(dev).to(torch.bfloat16)
    W = torch.from_numpy(x["W"]).to(dev).to(torch.bfloat16)
    del x
    chunk = args.chunk or w.chunk
    h = ckl.ChunkedKL(w.V, w.d, w.K, max_chunk=chunk, device=dev)
    n = ctypes.c_size_t()
    ckl._check(ckl.lib().ckl_topk_workspace_bytes(h._h, w.T, chunk, ctypes.byref(n)), "ws")
    ws = torch.empty(max(1, n.value), dtype=torch.uint8, device=dev)
    for _ in range(max(1, args.warmup)):
        h.topk_cache(H, W, chunk=chunk, workspace=ws, sync=False)
    stream = torch.cuda.current_stream(dev)
    n_chunks = (w.T + chunk - 1) // chunk
    h.profile_enable(True, args.steps * 4 * n_chunks + 8)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    e0.record(stream)
    for _ in range(args.steps):
        ids, lg = h.topk_cache(H, W, chunk=chunk, workspace=ws, sync=False)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    h.sync_status()
    ms = e0.elapsed_time(e1) / args.steps
    kern = {k["name"]: round(k["total_ms"] / args.steps, 3) for k in h.profile_collect()}
    peaks, src = load_peaks()
    tf = 4.0 * w.T * w.V * w.d / (ms / 1e3) / 1e12
    print(json.dumps({"kind": "topk_cache", "workload": w.name, "T": w.T, "V": w.V, "d": w.d,
                      "K": w.K, "chunk": chunk, "steps": args.steps, "ms_per_pass": ms,
                      "tokens_per_s": w.T / (ms / 1e3), "tflops_executed": tf,
                      "frac_of_sustained_bf16": tf / peaks["bf16_tflops_sustained"], "peak_source": src,
                      "workspace_mib": ws.numel() / 2**20, "kernel_ms_per_pass": kern}),
          flush=True)
    h.close()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="bf16_32k")
    ap.add_argument("--chunk", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-compare", action="store_true",
                    help="skip the pages' two other loss forms on this workload's inputs (N = 1)")
    ap.add_argument("--sweep", action="store_true",
                    help="256K workload: throughput vs chunk and peak memory vs T (extra JSON lines)")
    ap.add_argument("--sweep-steps", type=int, default=3)
    ap.add_argument("--compare", action="store_true",
                    help="the pages' Full Dense KL and Forward-Chunked Loss in plain PyTorch beside "
                         "this library: peak memory and step time vs T (extra JSON lines)")
    ap.add_argument("--compare-tokens", type=lambda v: [int(t) for t in v.split(",")],
                    default=[4096, 8192, 16384, 32768])
    ap.add_argument("--compare-steps", type=int, default=3)
    ap.add_argument("--graph-compare", action="store_true",
                    help="the workload's step eager vs replayed from a CUDA graph (extra JSON line)")
    ap.add_argument("--topk-cache", action="store_true",
                    help="time the teacher top-K cache builder on the workload's shape instead")
    ap.add_argument("--recompute", action="store_true",
                    help="form the logits again in the backward instead of keeping exp(z)")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        print("note: fewer than 3 warm-up steps", file=sys.stderr)

    from chunked_kl_loss_logits_b200.workloads import WORKLOADS
    w = WORKLOADS[args.workload]
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus and rank == 0:
        print(f"note: --gpus {args.gpus} but WORLD_SIZE={world}; using WORLD_SIZE", file=sys.stderr)

    if args.impl == "reference":
        run_reference(args, w, rank, world)
        return
    if args.sweep:
        run_sweep(args, w)
        return
    if args.topk_cache:
        run_topk_cache(args, w)
        return
    if args.graph_compare:
        run_graph_compare(args, w)
        return
    if args.compare:
        run_compare(args, w)
        return
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    try:
        run_ours(args, w, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
