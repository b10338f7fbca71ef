"""bench.py on the CPU: the multi-rank timing contract (two gloo ranks), the
reference arm, and the roofline arithmetic of the JSON line.

One process per GPU solves its own layer each step (weak scaling, no collective
on the data path); the job's time is the slowest rank's, and the metric counts
every rank's layers.
"""

import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch.distributed as dist

    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        slowest = bench.max_over_ranks(10.0 + 5.0 * rank, dist, "cpu")
        q.put((rank, slowest, bench.job_ms_per_layer(slowest, 3, world)))
    finally:
        dist.destroy_process_group()


def test_two_ranks_report_the_slowest_rank_over_all_layers():
    mp = pytest.importorskip("torch.multiprocessing")
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # rank 0 ran for 10 ms, rank 1 for 15 ms: both see 15 ms, and the job solved
    # 3 steps x 2 ranks = 6 layers in it
    assert results == [(0, 15.0, 2.5), (1, 15.0, 2.5)]


def test_single_process_needs_no_group():
    import bench
    assert bench.max_over_ranks(7.0, None, "cpu") == 7.0
    assert bench.job_ms_per_layer(12.0, 4, 1) == 3.0


def test_reference_arm_runs_on_rank_zero_only(capsys):
    import bench
    from synth import workload

    class Args:
        steps, warmup, gpus = 1, 0, 2

    bench.run_reference(Args(), workload("tiny_128x256"), rank=1, world=2)
    assert capsys.readouterr().out == ""


def test_phase_rooflines_from_measured_phase_times():
    # The per-phase rooflines of the bench line: algorithmic work over the phase
    # time, against the measured peaks (checked here on the 4096-wide layer).
    import bench
    from synth import workload
    wl = workload("llama7b_q_proj_4096x4096")
    peaks = {"bf16_tflops": 1606.3, "bf16_tflops_sustained": 1367.3, "hbm_gbs": 6539.5}
    phases = {"hessian": 3.62, "damp_perm": 0.017, "factor_U": 2.18, "sweep": 1.18,
              "finalize_pack": 0.05}
    roof = bench.phase_rooflines(wl, phases, peaks, 1606.3)
    assert set(roof) == set(phases)
    h = roof["hessian"]
    assert h["unit"] == "TFLOP/s" and h["peak"] == 1606.3
    assert h["achieved"] == pytest.approx(262144 * 4096 * 4097 / 3.62e-3 / 1e12, rel=1e-3)
    u = roof["factor_U"]
    assert u["peak"] == pytest.approx(1606.3 * 1.1 / 2.25 / 3, rel=1e-3)
    assert u["achieved"] == pytest.approx(2 * 4096 ** 3 / 3 / 2.18e-3 / 1e12, rel=1e-3)
    s = roof["sweep"]
    assert s["achieved"] == pytest.approx(4096 * 4096 * (4096 - 128) / 1.18e-3 / 1e12, rel=1e-3)
    f = roof["finalize_pack"]
    assert f["unit"] == "GB/s" and 0 < f["frac"] < 1
    assert bench.phase_rooflines(wl, {"hessian": 0.0}, peaks, 1606.3) == {}


@pytest.mark.parametrize("r,d,B,S", [(8, 1024, 128, 1024), (16, 4096, 128, 1024),
                                     (4, 1152, 64, 512), (3, 640, 32, 256)])
def test_sweep_flops_match_the_deferred_update_schedule(r, d, B, S):
    # The sweep's tensor work is the deferred trailing updates: inside each
    # superblock of S columns, block [j0, j1) updates the superblock's later
    # columns; each superblock then updates everything after it.  Summed over
    # that schedule, 2 r (j1 - j0) (end - j1) flops add up to r d (d - B): the
    # figure the bench line divides by the sweep's time.
    import bench
    from synth import Workload
    total = 0
    for s0 in range(0, d, S):
        s1 = min(d, s0 + S)
        for j0 in range(s0, s1, B):
            j1 = min(s1, j0 + B)
            total += 2 * r * (j1 - j0) * (s1 - j1)
        total += 2 * r * (s1 - s0) * (d - s1)
    assert total == r * d * (d - B)
    wl = Workload("t", r, d, 1, 4, -1, False, 1.0, 0.0, 1.0, 0.02, block=B)
    assert bench.phase_work(wl)["sweep"][1] * 1e12 == pytest.approx(total, rel=1e-12)


def test_tensor_peak_follows_the_sampled_clock():
    import bench
    peaks = {"bf16_tflops": 1606.3, "bf16_tflops_sustained": 1367.3}
    p, why = bench.tensor_peak(peaks, {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0})
    assert p == 1606.3 and "burst" in why
    p, why = bench.tensor_peak(peaks, {"sm_mhz": 1305.0, "sm_max_mhz": 1965.0})
    assert p == 1367.3 and "sustained" in why
    p, why = bench.tensor_peak(peaks, None)
    assert p == 1367.3
    p, why = bench.tensor_peak({}, None)
    assert "fallback" in why


@pytest.mark.parametrize("name", ["llama7b_q_proj_4096x4096", "opt175b_fc2_12288x49152"])
def test_recorded_hessian_traffic_is_for_the_current_kernel(name):
    # The DRAM bytes the bench reports for the Hessian come from an ncu capture of
    # the kernel as it is now: a change to its sources voids them (reported as
    # null) until they are captured again, and this test says so.
    import bench
    from synth import workload
    wl = workload(name)
    t = bench._traffic(wl)
    assert t is not None, "hessian_tc.cu or gptq_common.cuh changed since the capture"
    algorithmic = wl.x_bytes + 2 * 4 * wl.d * wl.d
    assert algorithmic <= t <= 10 * algorithmic


def test_cpu_sample_extrapolates_each_phase_by_its_cost():
    # The bounded CPU sample of a layer is scaled phase by phase; on the tiny
    # layer the sample is the whole layer, so nothing is scaled up.
    import bench
    from synth import workload, workload_inputs
    wl = workload("tiny_128x256")
    X, W = workload_inputs(wl)
    n_s, d_s, r_s = bench.sample_sizes(wl, big=True)
    assert (n_s, d_s, r_s) == (wl.n, wl.d, wl.r)
    res = bench._oracle_sample(wl, X, W, n_s, d_s, r_s)
    assert set(res["phases_s"]) == {"hessian", "factor", "sweep", "pack"}
    assert res["ms_per_layer"] > 0 and "extrapolated" in res["sample"]


def test_reference_arm_prints_one_complete_json_line():
    # `bench.py --impl reference` times the float64 oracle on the host cores and
    # prints the same JSON line as the GPU arm plus "impl": "reference".
    out = subprocess.run(
        [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
         "tiny_128x256", "--steps", "1", "--warmup", "0"],
        capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr
    lines = [ln for ln in out.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    line = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["higher_is_better"] is False
    assert line["value"] > 0 and line["unit"] == "ms per layer"
    assert line["config"]["workload"] == "tiny_128x256"
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"]
    assert line["extrapolated"] is True and cb["extrapolated"] is True
    e2e = line["e2e"]
    assert e2e["value"] == line["value"] and e2e["h2d_bytes_per_step"] == 0


