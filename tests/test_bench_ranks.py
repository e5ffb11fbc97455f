"""The multi-GPU path of bench.py on CPU: two gloo ranks (no GPU).  Ranks are
independent replicas, so the only cross-rank steps are the barrier and the
max of the timings; the job's throughput counts every rank's work."""
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


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        dist.barrier()
        elapsed = [120.0, 150.0][rank]                  # each rank's own device time
        got = bench.max_over_ranks(elapsed, dist, torch.device("cpu"))
        out[rank] = got
    finally:
        dist.destroy_process_group()


def test_max_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    port = _free_port()
    mp.start_processes(_rank_main, args=(2, port, out), nprocs=2, start_method="spawn", join=True)
    assert out[0] == 150.0 and out[1] == 150.0


def test_single_process_is_identity_and_throughput_is_job_wide():
    assert bench.max_over_ranks(12.5, None, None) == 12.5
    one = bench.job_throughput(1, bench.STEP_FLOPS, 100, 97.29)
    two = bench.job_throughput(2, bench.STEP_FLOPS, 100, 97.29)
    assert two == pytest.approx(2 * one)
    assert one == pytest.approx(bench.STEP_FLOPS * 100 / 97.29e-3 / 1e12)
