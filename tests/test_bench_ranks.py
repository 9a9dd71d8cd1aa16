"""The multi-GPU bench path without GPUs: two gloo ranks on the CPU check the
cross-rank aggregation (max over ranks, whole-job throughput) and that only
rank 0 runs and prints the reference (CPU oracle) arm."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, out):
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        local_ms = [12.5, 20.0][rank]                 # rank 1 is the slower one
        total = bench.max_over_ranks(local_ms, dist, torch.device("cpu"))
        value = bench.job_tflops(world, 1e12, 4, total)
        out.put((rank, total, value))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_ranks_take_the_slowest_rank_and_count_both_replicas():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, total, value in res:
        assert total == 20.0                          # both ranks see the max
        assert value == pytest.approx(2 * 1e12 * 4 / 20e-3 / 1e12)


def test_single_rank_aggregation_is_the_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(7.5, None, torch.device("cpu")) == 7.5
    assert bench.job_tflops(1, 2e12, 2, 4.0) == pytest.approx(1000.0)


def test_reference_arm_runs_on_rank_zero_only(capsys):
    sys.path.insert(0, ROOT)
    import bench

    class Args:
        gpus, steps, warmup = 2, 1, 0

    bench.run_reference(Args, rank=1, world=2)        # returns at once, prints nothing
    assert capsys.readouterr().out == ""


def test_reference_arm_reports_the_same_config_keys(capsys, monkeypatch):
    # the driver compares the two arms' lines: the reference arm names the same
    # workload with the same config keys as ours (the CPU oracle itself is stubbed out)
    sys.path.insert(0, ROOT)
    import json

    import bench

    monkeypatch.setattr(bench, "cpu_oracle_sample",
                        lambda problems, budget_s=0.0, rows=1, prepared=None, nthreads=0: (1.0, 0.01, 4, "stub", None))

    class Args:
        gpus, steps, warmup = 2, 2, 1

    bench.run_reference(Args, rank=0, world=2)
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC and line["unit"] == bench.UNIT
    assert set(line["config"]) == {"workload", "global_batch", "per_gpu_batch", "parallelism", "l2"}
    assert line["config"]["workload"] == bench.WORKLOAD
    assert line["config"]["global_batch"] == 256 and line["config"]["parallelism"] == "replicas x2"
