"""CPU test of bench.py's multi-rank path with two gloo ranks: the timings each rank
reports are reduced to the maximum over ranks on every rank, and the whole-job value
is N x the per-rank work over that time (replicas, weak scaling)."""

import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, results):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r reports (10 + r) ms per step and (5 - r) ms per kernel launch
        ms, kms = bench.max_over_ranks([10.0 + rank, 5.0 - rank], "cpu", world)
        results[rank] = (ms, kms, bench.weak_scaling_tflops(2.0e12, world, ms))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_weak_scaling_value_two_gloo_ranks():
    world = 2
    manager = mp.get_context("spawn").Manager()
    results = manager.dict()
    mp.start_processes(_rank_main, args=(world, _free_port(), results), nprocs=world,
                       join=True, start_method="spawn")
    assert sorted(results.keys()) == [0, 1]
    for r in range(world):
        ms, kms, value = results[r]
        assert ms == 11.0 and kms == 5.0          # the slowest rank's numbers, on every rank
        assert value == pytest.approx(2 * 2.0e12 / 11e-3 / 1e12)


def test_single_rank_passthrough():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks([3.0, 4.0], "cpu", 1) == [3.0, 4.0]
    assert bench.weak_scaling_tflops(1e12, 1, 1.0) == pytest.approx(1000.0)


def test_roofline_peak_follows_the_timed_region():
    """A kernel timed inside a sub-second region is held to the burst bf16 peak; only a
    region of seconds (the length of the sustained measurement's loop) takes the
    sustained figure."""
    sys.path.insert(0, ROOT)
    import bench
    peaks = {"bf16_tflops": 1653.8, "bf16_tflops_sustained": 1383.1}
    assert bench.roofline_peak(peaks, 0.5) == ("bf16_tflops", 1653.8)
    assert bench.roofline_peak(peaks, 4.0) == ("bf16_tflops_sustained", 1383.1)


def test_job_flop_for_replicas_and_head_sharding():
    """Replicas: N copies of the workload. Heads: the one layer, whatever share of its
    heads each rank holds."""
    sys.path.insert(0, ROOT)
    import bench
    assert bench.job_flop(10.0, 40, 40, 4, "replicas") == 40.0
    assert bench.job_flop(10.0, 10, 40, 4, "heads") == 40.0
    assert bench.job_flop(14.0, 14, 40, 3, "heads") == 40.0
