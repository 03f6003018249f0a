"""The multi-rank path of the benchmark on CPU: two gloo ranks, each timing its own
independent layer (weak scaling, no collective in the data path); the job's time is the
slowest rank's, and the throughput counts every rank's weights."""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        bench._barrier(world)
        # rank r "took" 100 + 50 r ms for its 3 steps
        total = bench._max_over_ranks(100.0 + 50.0 * rank, world)
        rate = bench.aggregate_rate(1000.0, world, 3, total)
        bench._barrier(world)
        out.put((rank, total, rate))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_time_and_weak_scaling_rate():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r for r, _, _ in res] == [0, 1]
    for _, total, rate in res:
        assert total == 150.0  # the slowest rank
        assert rate == pytest.approx(1000.0 * 2 * 3 / 0.150)


def test_single_rank_rate_is_plain_throughput():
    import bench
    assert bench._max_over_ranks(12.5, 1) == 12.5
    assert bench.aggregate_rate(5120 * 5120, 1, 10, 100.0) == pytest.approx(5120 * 5120 * 10 / 0.1)


def test_cpu_baseline_host_fields():
    """The oracle baseline records the host's CPU model and core count, and times the tiny
    layer's whole path single-threaded."""
    import bench
    host = bench._host_cpu()
    assert host["nproc"] >= 1
    tiny = bench._oracle_tiny_single_thread(reps=1)
    assert tiny["threads"] == 1 and tiny["s_per_step"] > 0 and tiny["weights_per_s"] > 0
    assert "W [64, 128]" in tiny["workload"]


def test_bench_line_carries_the_contract_keys():
    """The JSON line's keys and types (built from stand-in measurements); the dominant kernel's
    DRAM traffic comes from its committed profile, or is null once the kernel source changed."""
    import json
    import types

    import bench
    import workloads as wl
    cfg = wl.CONFIGS[1]
    args = types.SimpleNamespace(steps=10, warmup=3)
    peaks = dict(bench._peaks(), tf32_tflops=800.0, fp64_tflops=37.0)
    kernels = {"syrk": {"achieved": 1000.0, "ms_per_step": 0.2, "launches_per_step": 1.0, "ms_total": 0.4,
                        "work_total": 4.3e11, "launches_total": 2},
               "tf32_gemm": {"achieved": 120.0, "ms_per_step": 1.1, "launches_per_step": 39.0, "ms_total": 2.2,
                             "work_total": 2.6e11, "launches_total": 78}}
    e2e = {"value": 2.0e9, "unit": "weights/s", "h2d_bytes_per_step": 1, "d2h_bytes_per_step": 1}
    clocks = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": []}
    line = bench.build_line(args, cfg, 1, 2.8e9, 9.3, [0.2], [9.0], [0.03], [0.03], 900.0, 7.9e7, 1.3e8,
                            peaks, e2e, 394, clocks, ("f64_gemm_64", 33.0, 6.7e11, 40), kernels,
                            {"fp64_tflops": 37.0})
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "roofline", "e2e", "gpu_launches", "clocks"):
        assert key in line, key
    assert line["unit"] == "weights/s" and line["higher_is_better"] is True and line["scaling"] == "weak"
    assert "workload" in line["config"] and "model" not in line["config"]
    roof = line["roofline"]
    for key in ("bound", "achieved", "peak", "unit", "frac", "traffic"):
        assert key in roof, key
    assert roof["frac"] == pytest.approx(roof["achieved"] / roof["peak"])
    assert roof["peak"] == 37.0  # the fp64 rate measured in the run, not a nominal ratio
    assert roof["achieved"] == pytest.approx(6.7e11 / 0.033 / 1e12)
    i8 = bench.class_roofline("i8x_gemm", 10.0, 1e12, 4, 10, dict(peaks, int8_tops=3000.0), cfg)
    assert i8["unit"] == "TOP/s" and i8["achieved"] == pytest.approx(28 * 1e12 / 0.01 / 1e12)
    assert i8["frac"] == pytest.approx(i8["achieved"] / 3000.0)
    assert line["update_roofline"]["tf32_tflops"] == 800.0
    assert roof["traffic"] is None or roof["traffic"] > 0
    assert line["gpu_launches"] == 3940
    json.dumps(line)


def test_dominant_class_is_ranked_net_of_launch_processing():
    """A class of many short launches does not outrank a class of few long ones on the launch
    processing its per-launch event pairs hold; without the net figure the raw time decides; a
    dominant class with many launches per step is timed outside the headline steps, and the line
    says where it was timed."""
    import types

    import bench
    import workloads as wl
    kernels = {"f64_gemm_64": {"ms_per_step": 1.83, "ms_net_per_step": 0.94, "launches_per_step": 144.0},
               "i8x_gemm": {"ms_per_step": 1.52, "ms_net_per_step": 1.45, "launches_per_step": 12.0},
               "leaf": {"ms_per_step": 1.54, "ms_net_per_step": 1.29, "launches_per_step": 40.0}}
    assert bench.dominant_class(kernels) == "i8x_gemm"
    raw = {k: {kk: vv for kk, vv in v.items() if kk != "ms_net_per_step"} for k, v in kernels.items()}
    assert bench.dominant_class(raw) == "f64_gemm_64"
    assert bench.dominant_class({}) == "f64_gemm_64"
    assert 12 <= bench.MAX_INLINE_TIMED_LAUNCHES < 40
    cfg = wl.CONFIGS[1]
    args = types.SimpleNamespace(steps=10, warmup=3)
    peaks = dict(bench._peaks(), tf32_tflops=800.0, fp64_tflops=37.0, int8_tops=3000.0)
    clocks = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": []}
    e2e = {"value": 2.0e9, "unit": "weights/s", "h2d_bytes_per_step": 1, "d2h_bytes_per_step": 1}
    for inline, where in ((True, "inside the timed region"), (False, "second pass")):
        line = bench.build_line(args, cfg, 1, 2.8e9, 9.3, [0.2], [9.0], [0.03], [0.03], 900.0, 7.9e7, 1.3e8,
                                peaks, e2e, 249, clocks, ("leaf", 15.0, 1e9, 400), {}, {}, inline, 6.1)
        assert where in line["roofline"]["timing"]
        assert line["roofline"]["launch_overhead_us"] == 6.1


def test_reference_arm_times_what_it_reports():
    """The oracle arm on the tiny layer: the steps it reports are the steps it timed (their
    total fits inside the call's wall time), and its workload string is the GPU arm's."""
    import time
    import types

    import bench
    import workloads as wl
    args = types.SimpleNamespace(steps=2, warmup=1, config=0)
    t0 = time.perf_counter()
    line = bench.run_reference(args)
    wall = time.perf_counter() - t0
    assert line["impl"] == "reference" and line["steps"] == 2 and line["value"] > 0
    assert line["ms_per_step"] * line["steps"] / 1e3 <= wall
    assert line["config"]["workload"] == bench.workload_string(wl.CONFIGS[0])
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == line["value"] and cb["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0
