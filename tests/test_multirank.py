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
