#!/usr/bin/env python3
"""Benchmark: milliseconds per layer for the GPTQ layer solve on B200.

One step = one layer: H = 0, H += 2 X^T X (tensor cores), then the solve
(damping, Cholesky factor and inverse, column sweep with lazy trailing updates,
unpermute, loss, int32 packing).  Inputs are resident in HBM before the timed
region; X (6.4 GB for the default OPT-175B fc2 layer, 12288 x 49152 with 65536
tokens) is larger than L2, so nothing is reused between steps through the
cache.

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
DEFAULT_WORKLOAD = "opt175b_fc2_12288x49152"


def _args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=None,
                   help="timed steps (default: about half a minute of layers)")
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--e2e-steps", type=int, default=3)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--gemm-pair", action="store_true",
                   help="run products of two or more row tiles on CTA pairs")
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


# DRAM bytes (read + write) of one full-size launch of the Hessian kernel, from a one-pass
# ncu capture of the same workload.  Valid only for the kernel source it was taken on:
# reported as null as soon as the sources hash differently.
KERNEL_TRAFFIC = {
    "llama7b_q_proj_4096x4096": {
        "kernel": "hessian_tc_kernel",
        "sources": ["post_weight_quantization_19_b200/csrc/hessian_tc.cu",
                    "post_weight_quantization_19_b200/csrc/gptq_common.cuh"],
        "sha256": "c1316476f1761699e7b737b98978fa5e2f66baf5e0da481d69f9379a7422d40c",
        "bytes": 4269406976 + 42836480,
    },
    "opt175b_fc2_12288x49152": {
        "kernel": "hessian_tc_kernel",
        "sources": ["post_weight_quantization_19_b200/csrc/hessian_tc.cu",
                    "post_weight_quantization_19_b200/csrc/gptq_common.cuh"],
        "sha256": "c1316476f1761699e7b737b98978fa5e2f66baf5e0da481d69f9379a7422d40c",
        "bytes": 175541137408 + 9743772160,
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

def _cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def sample_sizes(wl, big: bool) -> tuple[int, int, int]:
    """(tokens, features, rows) of the bounded CPU sample: a leading block of the layer."""
    if big:
        return min(wl.n, 16384), min(wl.d, 8192), min(wl.r, 256)
    return min(wl.n, 8192), min(wl.d, 4096), min(wl.r, 128)


def _oracle_sample(wl, X, W, n_s: int, d_s: int, r_s: int) -> dict:
    """Time the float64 oracle on the leading n_s x d_s block of X and r_s x d_s of W,
    then extrapolate each phase to the whole layer by its cost model:
    Hessian n*d*(d+1); factor d^3; sweep a*d + b*d^2 per row (fitted from the
    sample at d_s and d_s/2: the column loop and the deferred updates), times
    r/r_s; packing r*d."""
    import oracle

    Xs = np.ascontiguousarray(X[:n_s, :d_s])
    Ws = np.ascontiguousarray(W[:r_s, :d_s])
    t0 = time.perf_counter()
    H = oracle.hessian(Xs)
    t1 = time.perf_counter()
    Hd, _ = oracle.dampen(H, wl.damp)
    perm = oracle.act_order_perm(H) if wl.act_order else np.arange(d_s)
    U = oracle.inverse_upper_cholesky(Hd[np.ix_(perm, perm)])
    t2 = time.perf_counter()
    g = wl.group if wl.group == -1 or d_s % wl.group == 0 else -1
    codes, *_ = oracle.gptq_sweep(Ws[:, perm], U, wl.bits, g, wl.block)
    t3 = time.perf_counter()
    h2 = d_s // 2
    oracle.gptq_sweep(Ws[:, perm][:, :h2], U[:h2, :h2], wl.bits, g if g == -1 or h2 % g == 0
                      else -1, wl.block)
    t4 = time.perf_counter()
    oracle.pack_rows(codes, wl.bits)
    t5 = time.perf_counter()
    th, tf, ts, ts2, tp = t1 - t0, t2 - t1, t3 - t2, t4 - t3, t5 - t4
    # sweep(d) = a d + b d^2 through (d_s/2, ts2) and (d_s, ts)
    b = max((ts - 2.0 * ts2) / (d_s * d_s / 2.0), 0.0)
    a = max((ts - b * d_s * d_s) / d_s, 0.0)
    d, n, r = wl.d, wl.n, wl.r
    phases = {
        "hessian": th * (n / n_s) * (d * (d + 1.0)) / (d_s * (d_s + 1.0)),
        "factor": tf * (d / d_s) ** 3,
        "sweep": (a * d + b * d * d) * (r / r_s),
        "pack": tp * (r / r_s) * (d / d_s),
    }
    return {"ms_per_layer": 1e3 * sum(phases.values()), "measured_s": t5 - t0,
            "phases_s": phases,
            "sample": (f"float64 numpy oracle on a leading block: Hessian of {n_s} tokens x {d_s} "
                       f"features (x{n / n_s:g} tokens, x{(d * (d + 1.0)) / (d_s * (d_s + 1.0)):.4g} "
                       f"features^2), damping+inverse+Cholesky at {d_s} (x{(d / d_s) ** 3:.4g}, "
                       f"d^3), sweep of {r_s} rows at {d_s} and {h2} columns fitted to a*d+b*d^2 "
                       f"and scaled to {d} columns x {r / r_s:g} rows, packing x{r / r_s * d / d_s:.4g}"
                       f"; {t5 - t0:.1f} s measured, the rest extrapolated")}


def cpu_baseline(wl, X, W) -> dict:
    n_s, d_s, r_s = sample_sizes(wl, big=True)
    res = _oracle_sample(wl, X, W, n_s, d_s, r_s)
    return {"value": round(res["ms_per_layer"], 3), "unit": "ms per layer", "cores": _cores(),
            "kind": "oracle", "extrapolated": True, "sample": res["sample"],
            "phases_s": {k: round(v, 3) for k, v in res["phases_s"].items()}}


def run_reference(args, wl, rank: int, world: int):
    if rank != 0:
        return
    n_s, d_s, r_s = sample_sizes(wl, big=False)
    X, W = workload_inputs(wl, n=n_s)
    steps = args.steps if args.steps is not None else 10
    for _ in range(args.warmup):
        _oracle_sample(wl, X, W, n_s, d_s, r_s)
    vals, wall, res = [], 0.0, None
    for _ in range(steps):
        res = _oracle_sample(wl, X, W, n_s, d_s, r_s)
        vals.append(res["ms_per_layer"])
        wall += res["measured_s"]
    value = float(np.mean(vals))
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "ms per layer",
        "n_gpus": args.gpus, "steps": steps, "warmup": args.warmup,
        "ms_per_step": round(value, 3), "higher_is_better": False, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": _config(wl),
        "extrapolated": True,
        "cpu_baseline": {"value": round(value, 3), "unit": "ms per layer", "cores": _cores(),
                         "kind": "oracle", "extrapolated": True,
                         "sample": "each step: " + res["sample"],
                         "measured_s_per_step": round(wall / steps, 3)},
        "e2e": {"value": round(value, 3), "unit": "ms per layer", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ rooflines

# Nominal dense tensor rates (PFLOP/s) used to carry the measured bf16 peak over
# to another operand type: tf32 is 1.1 against 2.25 for fp16/bf16.
TF32_OVER_BF16 = 1.1 / 2.25


def tensor_peak(peaks: dict, clocks: dict | None) -> tuple[float, str]:
    """Measured bf16 tensor peak: the burst figure while the sampled SM clock held
    its maximum during the timed region, else the sustained (power-capped) one."""
    burst = peaks.get("bf16_tflops")
    sust = peaks.get("bf16_tflops_sustained")
    if burst is None or sust is None:
        return 1590.0, "fallback burst (no MEASURED_PEAKS.json)"
    sm, smax = (clocks or {}).get("sm_mhz"), (clocks or {}).get("sm_max_mhz")
    if sm and smax and sm >= 0.97 * smax:
        return float(burst), f"measured burst: the SM clock held {sm:.0f} of {smax:.0f} MHz"
    return float(sust), (f"measured sustained: the SM clock median was {sm} of {smax} MHz"
                         if sm else "measured sustained: no clock samples")


def phase_work(wl) -> dict:
    """Algorithmic work of each phase of one layer: (unit, amount, kind).

    hessian: n*d*(d+1) flop (the symmetric product, upper triangle credited);
    factor_U: 2 d^3 / 3 flop (Cholesky and triangular inverse); sweep: r*d*(d-B)
    flop of the deferred trailing updates that dominate it (the sum over blocks
    of 2 r B (d - end of block)); damp_perm and finalize_pack: the bytes they must
    move.  Flops of the fp32 phases are fp32-equivalent."""
    r, d, n, B = wl.r, wl.d, wl.n, wl.block
    G = 1 if wl.group == -1 else d // wl.group
    return {
        "hessian": ("TFLOP/s", float(n) * d * (d + 1) / 1e12, "fp16"),
        "damp_perm": ("GB/s", 8.0 * d * (d if wl.act_order else 1) / 1e9, "hbm"),
        "factor_U": ("TFLOP/s", 2.0 * d ** 3 / 3.0 / 1e12, "3xtf32"),
        "sweep": ("TFLOP/s", float(r) * d * max(d - B, 0) / 1e12, "3xtf32"),
        "finalize_pack": ("GB/s", (r * d * (4 + 4 + 1 + wl.bits / 8.0) + 8.0 * r * G) / 1e9, "hbm"),
    }


def phase_rooflines(wl, phases_ms: dict, peaks: dict, tc_peak: float) -> dict:
    """Each phase of one layer against the roofline of its algorithmic work:
    fp16 contractions against the bf16 tensor peak; the fp32 products (three
    TF32 products per fp32 product on the tensor cores) against a third of the
    TF32 peak; byte-bound phases against the measured HBM copy rate."""
    hbm = float(peaks.get("hbm_gbs", 6650.0))
    peak_of = {"fp16": tc_peak, "3xtf32": tc_peak * TF32_OVER_BF16 / 3.0, "hbm": hbm}
    out = {}
    for name, (unit, amount, kind) in phase_work(wl).items():
        ms = phases_ms.get(name)
        if not ms or ms <= 0:
            continue
        achieved = amount / (ms * 1e-3)
        out[name] = {"achieved": round(achieved, 2), "peak": round(peak_of[kind], 1), "unit": unit,
                     "frac": round(achieved / peak_of[kind], 4), "work": amount,
                     "ms": round(ms, 4)}
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

def default_steps(wl) -> int:
    """About half a minute of timed layers: 60 steps of the 4096-wide layers, fewer of
    the wider ones."""
    return 10 if wl.d >= 16384 else (30 if wl.d >= 8192 else 60)


def run_ours(args, wl, rank: int, world: int, dist):
    import torch

    import post_weight_quantization_19_b200 as g

    g.gptq_set_gemm_pair(args.gemm_pair)
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    steps = args.steps if args.steps is not None else default_steps(wl)
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
    names = ["damp_perm", "factor_U", "sweep", "finalize_pack"]

    def step():
        """One layer; returns (loss, Hessian ms, phase ms) -- every time on the device,
        with CUDA events on the launching stream (the solve's phase events are
        nodes of its replayed graph)."""
        H.zero_()
        h_start.record(stream)
        g.gptq_hessian_accumulate(Xd, H, stream=stream)
        h_end.record(stream)
        res = g.gptq_quantize_layer(Wd, H, bits=wl.bits, group=wl.group, block=wl.block,
                                    damp=wl.damp, act_order=wl.act_order, g_idx=g_idx,
                                    workspace=ws, outputs=outs, stream=stream)
        # quantize_layer returns after synchronising its stream
        return res["loss"], h_start.elapsed_time(h_end), g.gptq_last_phase_ms()

    g.gptq_set_phase_timing(True)
    for _ in range(max(args.warmup, 1)):
        step()

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
    h_ms, ph_ms, loss = [], [], None
    t_start.record(stream)
    for _ in range(steps):
        loss, hm, ph = step()
        h_ms.append(hm)
        ph_ms.append(ph)
    t_end.record(stream)
    torch.cuda.synchronize(dev)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize(dev)
    launches = g.gptq_launch_count() - launches0
    clocks = sampler.stop()
    g.gptq_set_phase_timing(False)
    elapsed = max_over_ranks(t_start.elapsed_time(t_end), dist, dev)
    ms_per_step = elapsed / steps
    value = job_ms_per_layer(elapsed, steps, world)

    # end to end through the host-buffer entry point
    e2e = None
    if args.e2e_steps > 0:
        Xh = torch.from_numpy(X).pin_memory()
        Wh = torch.from_numpy(W).pin_memory()
        del Xd
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
    tc_peak, peak_src = tensor_peak(peaks, clocks)
    phases_ms = {"hessian": round(float(np.mean(h_ms)), 4)}
    for i, nm in enumerate(names):
        vals = [p[i] for p in ph_ms if len(p) > i and p[i] > 0]
        if vals:
            phases_ms[nm] = round(float(np.mean(vals)), 4)
    pr = phase_rooflines(wl, phases_ms, peaks, tc_peak)
    if "hessian" in pr:   # DRAM bytes of the one-launch phase, when captured on this source
        pr["hessian"]["traffic"] = _traffic(wl)
    # The dominant kernel: the Hessian is one launch per step; the factorisation and
    # the sweep are phases whose tensor work is the 3xTF32 GEMM (with the leaves /
    # in-block sweep kernels on their critical path), timed by the phase events.
    kernel_of = {"hessian": "hessian_tc_kernel",
                 "factor_U": "gemm_pair_*_kernel / gemm_tc_kernel (factorisation phase: "
                             "leaf_kernel chain + 3xTF32 GEMMs)",
                 "sweep": "gemm_pair_*_kernel / gemm_tc_kernel (sweep phase: trailing-update "
                          "GEMMs + sweep_block_kernel)"}
    dom = max((k for k in kernel_of if k in pr), key=lambda k: pr[k]["ms"])
    dp = pr[dom]
    roofline = {"bound": "tensor", "kernel": kernel_of[dom], "phase": dom,
                "achieved": dp["achieved"], "peak": dp["peak"], "unit": "TFLOP/s",
                "frac": dp["frac"], "traffic": _traffic(wl) if dom == "hessian" else None,
                "peak_source": peak_src + ("; fp16 runs at the bf16 rate" if dom == "hessian" else
                                           "; TF32 = bf16 x 1.1/2.25 (nominal ratio), three TF32 "
                                           "products per fp32-equivalent product"),
                "work_per_step": dp["work"] * 1e12, "avg_ms": dp["ms"]}
    line = {
        "metric": METRIC, "value": round(value, 4), "unit": "ms per layer", "n_gpus": world,
        "steps": steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None,
        "dtype": "f16 in / f32 accumulate (Hessian); f32 solve (3xTF32 tensor-core products)",
        "data": "synthetic", "config": _config(wl),
        "roofline": roofline,
        "phases_ms": phases_ms,
        "phase_roofline": pr,
        "loss": loss,
        "gpu_launches": int(launches),
        "gemm_pair": {"enabled": bool(args.gemm_pair), "form": g.gptq_gemm_pair_form()[0]},
        "clocks": clocks,
        "e2e": e2e,
    }
    if not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl, X, W)
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
