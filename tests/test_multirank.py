"""The job across ranks (bench.py), on CPU with gloo: the job's time is the slowest rank's,
its throughput counts every rank's steps, and only rank 0 runs the oracle arm."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, times, out):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        t = bench.max_over_ranks(times[rank])
        out.put((rank, t, bench.job_throughput(10, world, 20, t)))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_slowest_rank_sets_the_job_time(world):
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    times = [0.5 + 0.25 * r for r in range(world)]
    mp.start_processes(_rank_main, args=(world, _free_port(), times, out), nprocs=world,
                       join=True, start_method="spawn")
    got = sorted(out.get(timeout=60) for _ in range(world))
    for rank, t, v in got:
        assert t == max(times)                       # every rank agrees on the max
        assert v == pytest.approx(10 * world * 20 / max(times))


def test_single_process_is_unchanged():
    import bench
    assert bench.max_over_ranks(1.25) == 1.25
    assert bench.job_throughput(7, 1, 20, 2.0) == 70.0


def test_reference_arm_runs_on_rank_0_only(capsys):
    import argparse

    import bench
    args = argparse.Namespace(workload="tiny", steps=1, warmup=3, gpus=2)
    bench.run_reference(args, rank=1)                # other ranks exit without work
    assert capsys.readouterr().out == ""


def test_reference_arm_line(capsys):
    """The oracle arm prints one JSON line with the contract's keys, on the host cores."""
    import argparse
    import json

    import bench
    args = argparse.Namespace(workload="tiny", steps=1, warmup=3, gpus=1)
    bench.run_reference(args, rank=0)
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "layer-steps/s"
    assert line["metric"] == bench.METRIC and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"] == {"value": line["value"], "unit": "layer-steps/s",
                           "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_schedule_description():
    import bench
    from fp4_kv_cache_03_b200 import synth
    assert bench.schedule_of(synth.workload("decoder_step_128k").modes) == \
        "full, 3 reuse, " + ", ".join(["reindex, 3 reuse"] * 4)
    assert bench.schedule_of(("full",)) == "full"
