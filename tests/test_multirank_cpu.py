"""The multi-process host logic of bench.py on CPU: two gloo ranks.

bench.py --gpus N runs N independent replicas (the scan has no exchange step);
what crosses ranks is the timing: every rank takes the slowest rank's time and
the job's throughput counts the units of all ranks.  The reference arm runs on
rank 0 only.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, results):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        cpu = torch.device("cpu")
        ms = [3.5, 7.25][rank]                      # each rank's own timed region
        slowest = bench.max_over_ranks(ms, world, cpu)
        rate = bench.job_rate(world, 16384, 20, slowest)
        dist.barrier()
        results[rank] = (slowest, rate)
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_slowest_time_and_count_all_units():
    world = 2
    with mp.Manager() as mgr:
        results = mgr.dict()
        mp.start_processes(_worker, args=(world, _free_port(), results), nprocs=world,
                           start_method="spawn", join=True)
        got = dict(results)
    assert got[0] == got[1]
    slowest, rate = got[0]
    assert slowest == 7.25
    assert rate == pytest.approx(2 * 16384 * 20 / 7.25e-3)


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(1.5, 1, torch.device("cpu")) == 1.5
    assert bench.job_rate(1, 100, 10, 2.0) == pytest.approx(100 * 10 / 2e-3)


def test_reference_arm_runs_on_rank_zero_only(capsys):
    class Args:
        workload = "tiny_f32"
        ref_tokens = 8
        warmup = 3
        steps = 1
        gpus = 2
    bench.run_reference(Args, {}, rank=1)
    assert capsys.readouterr().out == ""
