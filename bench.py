#!/usr/bin/env python3
"""Benchmark: milliseconds per layer for the GPTQ layer solve on B200.

One step = one layer: H = 0, H += 2 X^T X (tensor cores), then the solve
(damping, Cholesky factor and inverse, column sweep with lazy trailing updates,
unpermute, loss, int32 packing).  Inputs are resident in HBM before the timed
region; X (2.1 GB for the default workload) is larger than L2, so nothing is
reused between steps through the cache.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

With N > 1 (launched by torch.distributed.run) every rank solves its own layer
(layers are independent problems: weak scaling, no collective on the data
path); the timing is the max over ranks.  ``--impl reference`` times the float64
CPU oracle on a bounded sample of the same workload instead.

Prints one JSON line on rank 0.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from synth import WORKLOADS, workload, workload_inputs  # noqa: E402

METRIC = "ms per layer (Hessian+Cholesky+solve+pack) and % of tensor/HBM roofline"
DEFAULT_WORKLOAD = "llama7b_q_proj_4096x4096"


def _args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=60)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--e2e-steps", type=int, default=3)
    p.add_argument("--no-cpu-baseline", action="store_true")
    return p.parse_args()


def _config(wl) -> dict:
    return {
        "workload": wl.name, "r": wl.r, "d": wl.d, "n_tokens": wl.n, "bits": wl.bits,
        "group": wl.group, "block": wl.block, "act_order": wl.act_order, "damp": wl.damp,
        "inputs": "seeded synthetic (PCG64): X ~ N(0,1)*lognormal per channel with 0.1% x50 "
                  "outlier channels, W ~ N(0, sigma^2)",
        "l2": "inputs larger than L2 (X is %.2f GB)" % (wl.x_bytes / 1e9),
        "parallelism": "one independent layer per GPU",
    }


# DRAM bytes (read + write) of one full-size launch of the dominant kernel, from a one-pass
# ncu capture (profiles/hessian_tc_kernel_traffic.md).  Valid only for the kernel source it
# was taken on: reported as null as soon as the sources hash differently.
KERNEL_TRAFFIC = {
    "llama7b_q_proj_4096x4096": {
        "kernel": "hessian_tc_kernel",
        "sources": ["post_weight_quantization_19_b200/csrc/hessian_tc.cu",
                    "post_weight_quantization_19_b200/csrc/gptq_common.cuh"],
        "sha256": "53c32a78488a3a1be69bbb69f51edb36d0ae8754eef01037ae5f30d86b1c4e17",
        "bytes": 7386331136 + 51261184,
    },
}


def _traffic(wl) -> float | None:
    import hashlib

    rec = KERNEL_TRAFFIC.get(wl.name)
    if not rec or rec["bytes"] is None or rec["sha256"] is None:
        return None
    h = hashlib.sha256()
    for rel in rec["sources"]:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return float(rec["bytes"]) if h.hexdigest() == rec["sha256"] else None


def _peaks() -> dict:
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return json.load(f)
    except OSError:
        return {}


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""

    FIELDS = ["clocks.sm", "clocks.max.sm", "power.draw",
              "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]
    NAMES = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, bus_id: str | None):
        self.bus_id = bus_id
        self.proc = None
        self.lines: list[str] = []
        self.thread = None

    def start(self):
        cmd = ["nvidia-smi", "--query-gpu=" + ",".join(self.FIELDS),
               "--format=csv,noheader,nounits", "-lms", "100"]
        if self.bus_id:
            cmd[1:1] = ["-i", self.bus_id]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                                         text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self) -> dict | None:
        if not self.proc:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=5)
        sm, smax, reasons = [], [], set()
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) != len(self.FIELDS):
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
            except ValueError:
                continue
            for name, val in zip(self.NAMES, parts[3:]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax),
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------ CPU oracle leg

def _oracle_sample(wl, X, W, n_s: int, r_s: int) -> dict:
    """Time the float64 oracle on a bounded sample and scale each phase to the layer."""
    import oracle

    t0 = time.perf_counter()
    H = oracle.hessian(X[:n_s])
    t1 = time.perf_counter()
    Hd, _ = oracle.dampen(H, wl.damp)
    perm = oracle.act_order_perm(H) if wl.act_order else np.arange(wl.d)
    U = oracle.inverse_upper_cholesky(Hd[np.ix_(perm, perm)])
    t2 = time.perf_counter()
    codes, *_ = oracle.gptq_sweep(W[:r_s][:, perm], U, wl.bits, wl.group, wl.block)
    t3 = time.perf_counter()
    oracle.pack_rows(codes, wl.bits)
    t4 = time.perf_counter()
    ms = 1e3 * ((t1 - t0) * wl.n / n_s + (t2 - t1) + (t3 - t2) * wl.r / r_s
                + (t4 - t3) * wl.r / r_s)
    return {"ms_per_layer": ms, "measured_s": t4 - t0,
            "phases_s": [t1 - t0, t2 - t1, t3 - t2, t4 - t3]}


def _cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def cpu_baseline(wl, X, W, n_s: int, r_s: int) -> dict:
    res = _oracle_sample(wl, X, W, n_s, r_s)
    return {"value": round(res["ms_per_layer"], 3), "unit": "ms per layer", "cores": _cores(),
            "kind": "oracle",
            "sample": f"float64 numpy oracle: Hessian on {n_s} of {wl.n} tokens (x{wl.n / n_s:g}),"
                      f" full {wl.d}x{wl.d} damping+inverse+Cholesky, sweep+pack on {r_s} of "
                      f"{wl.r} rows (x{wl.r / r_s:g}); {res['measured_s']:.1f} s measured"}


def run_reference(args, wl, rank: int, world: int):
    if rank != 0:
        return
    n_s, r_s = min(wl.n, 8192), min(wl.r, 32)
    X, W = workload_inputs(wl, n=n_s)
    for _ in range(args.warmup):
        _oracle_sample(wl, X, W, n_s, r_s)
    vals, wall = [], 0.0
    for _ in range(args.steps):
        res = _oracle_sample(wl, X, W, n_s, r_s)
        vals.append(res["ms_per_layer"])
        wall += res["measured_s"]
    value = float(np.mean(vals))
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "ms per layer",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(value, 3), "higher_is_better": False, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": _config(wl),
        "cpu_baseline": {"value": round(value, 3), "unit": "ms per layer", "cores": _cores(),
                         "kind": "oracle",
                         "sample": f"each step: Hessian on {n_s} tokens (scaled x{wl.n / n_s:g}), "
                                   f"full d={wl.d} factor, sweep+pack on {r_s} rows (scaled "
                                   f"x{wl.r / r_s:g})"},
        "e2e": {"value": round(value, 3), "unit": "ms per layer", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ per-phase rooflines

def phase_rooflines(wl, phases_ms: dict, peaks: dict) -> dict:
    """Each phase of one layer against the roofline of its algorithmic work.

    hessian: n*d*(d+1) flop vs the sustained fp16 (bf16) tensor peak; factor_U:
    2 d^3 / 3 flop (Cholesky and triangular inverse) and sweep: r*d*(d-B) flop of
    the trailing updates that dominate it, both fp32-equivalent against a third of
    the TF32 peak (three TF32 products per fp32 product; TF32 is half the bf16 rate);
    damp_perm and finalize_pack: the bytes they must move vs the measured HBM copy
    rate.  The two latency-chain phases (factor_U, the in-block part of sweep) are
    not expected to approach their bound.
    """
    r, d, n, B = wl.r, wl.d, wl.n, wl.block
    tc = float(peaks.get("bf16_tflops_sustained", 1400.0))
    hbm = float(peaks.get("hbm_gbs", 6650.0))
    tf32x3 = tc / 2.0 / 3.0
    G = 1 if wl.group == -1 else d // wl.group
    work = {
        "hessian": ("TFLOP/s", float(n) * d * (d + 1) / 1e12, tc),
        "damp_perm": ("GB/s", 8.0 * d * (d if wl.act_order else 1) / 1e9, hbm),
        "factor_U": ("TFLOP/s", 2.0 * d ** 3 / 3.0 / 1e12, tf32x3),
        "sweep": ("TFLOP/s", 2.0 * r * d * max(d - B, 0) / 1e12, tf32x3),
        "finalize_pack": ("GB/s", (r * d * (4 + 4 + 1 + wl.bits / 8.0) + 8.0 * r * G) / 1e9, hbm),
    }
    out = {}
    for name, (unit, amount, peak) in work.items():
        ms = phases_ms.get(name)
        if not ms or ms <= 0:
            continue
        achieved = amount / (ms * 1e-3)
        out[name] = {"achieved": round(achieved, 2), "peak": round(peak, 1), "unit": unit,
                     "frac": round(achieved / peak, 4)}
    return out


# ------------------------------------------------------------------ multi-rank timing

def max_over_ranks(x: float, dist, device) -> float:
    """The largest per-rank value over the process group (a job takes as long as its
    slowest rank); ``dist`` is None for a single process."""
    if dist is None:
        return x
    import torch
    t = torch.tensor([x], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_ms_per_layer(elapsed_ms: float, steps: int, world: int) -> float:
    """Whole-job metric: the slowest rank's time over all layers the ranks processed
    (each rank solves one layer per step)."""
    return elapsed_ms / (steps * world)


# ------------------------------------------------------------------ GPU leg

def run_ours(args, wl, rank: int, world: int, dist):
    import torch

    import post_weight_quantization_19_b200 as g

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    X, W = workload_inputs(wl)
    r, d, n = wl.r, wl.d, wl.n
    G = 1 if wl.group == -1 else d // wl.group
    Xd = torch.from_numpy(X).to(dev)
    Wd = torch.from_numpy(W).to(dev)
    H = torch.empty((d, d), dtype=torch.float32, device=dev)
    ws = torch.empty(g.gptq_quantize_workspace_bytes(r, d, wl.bits, wl.group, wl.block,
                                                     wl.act_order), dtype=torch.uint8,
                     device=dev)
    outs = {"qweight": torch.empty((r, d * wl.bits // 32), dtype=torch.int32, device=dev),
            "scales": torch.empty((r, G), dtype=torch.float32, device=dev),
            "zeros": torch.empty((r, G), dtype=torch.int32, device=dev)}
    g_idx = torch.empty((d,), dtype=torch.int32, device=dev)
    stream = torch.cuda.Stream(dev)   # a capturable stream: the solve replays as a CUDA graph
    torch.cuda.set_stream(stream)
    h_start = torch.cuda.Event(enable_timing=True)
    h_end = torch.cuda.Event(enable_timing=True)

    def step(time_h: bool):
        H.zero_()
        if time_h:
            h_start.record(stream)
        g.gptq_hessian_accumulate(Xd, H, stream=stream)
        if time_h:
            h_end.record(stream)
        res = g.gptq_quantize_layer(Wd, H, bits=wl.bits, group=wl.group, block=wl.block,
                                    damp=wl.damp, act_order=wl.act_order, g_idx=g_idx,
                                    workspace=ws, outputs=outs, stream=stream)
        return res["loss"]

    for _ in range(max(args.warmup, 1)):
        step(False)
    # per-phase times (one extra untimed step with phase events on)
    g.gptq_set_phase_timing(True)
    h_start.record(stream)
    H.zero_()
    g.gptq_hessian_accumulate(Xd, H, stream=stream)
    h_end.record(stream)
    loss = g.gptq_quantize_layer(Wd, H, bits=wl.bits, group=wl.group, block=wl.block,
                                 damp=wl.damp, act_order=wl.act_order, g_idx=g_idx,
                                 workspace=ws, outputs=outs, stream=stream)["loss"]
    phases = g.gptq_last_phase_ms()
    phase_h = h_start.elapsed_time(h_end)
    g.gptq_set_phase_timing(False)

    bus = None
    try:
        p = torch.cuda.get_device_properties(dev)
        bus = "%08X:%02X:%02X.0" % (p.pci_domain_id, p.pci_bus_id, p.pci_device_id)
    except Exception:
        bus = None
    sampler = ClockSampler(bus)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize(dev)
    sampler.start()
    time.sleep(0.3)
    launches0 = g.gptq_launch_count()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    h_ms = []
    t_start.record(stream)
    for _ in range(args.steps):
        step(True)
        h_ms.append(h_start.elapsed_time(h_end))
    t_end.record(stream)
    torch.cuda.synchronize(dev)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize(dev)
    launches = g.gptq_launch_count() - launches0
    clocks = sampler.stop()
    elapsed = max_over_ranks(t_start.elapsed_time(t_end), dist, dev)
    ms_per_step = elapsed / args.steps
    value = job_ms_per_layer(elapsed, args.steps, world)

    # end to end through the host-buffer entry point
    e2e = None
    if args.e2e_steps > 0:
        Xh = torch.from_numpy(X).pin_memory()
        Wh = torch.from_numpy(W).pin_memory()
        hws = torch.empty(g.gptq_layer_host_workspace_bytes(r, d, n, wl.bits, wl.group,
                                                            wl.block, wl.act_order),
                          dtype=torch.uint8, device=dev)
        host_out = {k: torch.empty(v.shape, dtype=v.dtype).pin_memory() for k, v in outs.items()}
        host_out["g_idx"] = torch.empty((d,), dtype=torch.int32).pin_memory()
        g.gptq_solve_layer_host(Xh, Wh, bits=wl.bits, group=wl.group, block=wl.block,
                                damp=wl.damp, act_order=wl.act_order, dev_workspace=hws,
                                outputs=host_out, stream=stream)
        if dist is not None:
            dist.barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.e2e_steps):
            g.gptq_solve_layer_host(Xh, Wh, bits=wl.bits, group=wl.group, block=wl.block,
                                    damp=wl.damp, act_order=wl.act_order, dev_workspace=hws,
                                    outputs=host_out, stream=stream)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        e_ms = max_over_ranks(e0.elapsed_time(e1), dist, dev)
        out_bytes = sum(v.numel() * v.element_size() for v in host_out.values()) + 8
        e2e = {"value": round(job_ms_per_layer(e_ms, args.e2e_steps, world), 3),
               "unit": "ms per layer",
               "h2d_bytes_per_step": int(X.nbytes + W.nbytes), "d2h_bytes_per_step": int(out_bytes)}

    if rank != 0:
        return
    peaks = _peaks()
    h_avg = float(np.mean(h_ms))
    flops = float(n) * d * (d + 1)       # symmetric Hessian, upper triangle credited
    achieved = flops / (h_avg * 1e-3) / 1e12
    if "bf16_tflops_sustained" in peaks:
        peak, peak_src = float(peaks["bf16_tflops_sustained"]), "measured (sustained)"
    else:
        peak, peak_src = 1400.0, "fallback (sustained)"
    phases_ms = {"hessian": round(phase_h, 4), "damp_perm": round(phases[0], 4),
                 "factor_U": round(phases[1], 4), "sweep": round(phases[2], 4),
                 "finalize_pack": round(phases[3], 4)}
    line = {
        "metric": METRIC, "value": round(value, 4), "unit": "ms per layer", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None,
        "dtype": "f16 in / f32 accumulate (Hessian); f32 solve", "data": "synthetic",
        "config": _config(wl),
        "roofline": {"bound": "tensor", "kernel": "hessian_tc_kernel",
                     "achieved": round(achieved, 1), "peak": peak, "unit": "TFLOP/s",
                     "frac": round(achieved / peak, 4), "traffic": _traffic(wl),
                     "peak_source": peak_src + " bf16 cuBLAS peak; fp16 runs at the same rate",
                     "flops_per_launch": flops, "avg_launch_ms": round(h_avg, 4)},
        "phases_ms": phases_ms,
        "phase_roofline": phase_rooflines(wl, phases_ms, peaks),
        "loss": loss,
        "gpu_launches": int(launches),
        "clocks": clocks,
        "e2e": e2e,
    }
    if not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl, X, W, min(n, 8192), min(r, 32))
    print(json.dumps(line), flush=True)


def main():
    args = _args()
    wl = workload(args.workload)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        run_reference(args, wl, rank, world)
        return
    dist = None
    if world > 1:
        import datetime

        import torch
        import torch.distributed as tdist
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
        dist = tdist
    try:
        run_ours(args, wl, rank, world, dist)
    finally:
        if dist is not None:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
