"""Host logic of the multi-GPU benchmark path on CPU with gloo, world size 2:
each rank draws its own workload instance, the slowest rank's time is what
every rank reports, and the job throughput counts every rank's work."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from io_aware_exact_30_b200 import synth


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = 10.0 + 5.0 * rank  # rank 1 is the slow one
        mx = bench.reduce_max(local_ms, world)
        seed = bench.rank_seed(0, rank)
        q = synth.tensor(seed, synth.STREAM_Q, (1, 1, 8, 64))
        gathered = [None] * world
        dist.all_gather_object(gathered, q.tobytes())
        out[rank] = (mx, seed, gathered)
    finally:
        dist.destroy_process_group()


def test_two_rank_gloo_host_path():
    world, port = 2, _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, start_method="spawn", join=True)
    (mx0, s0, g0), (mx1, s1, g1) = out[0], out[1]
    assert mx0 == mx1 == 15.0
    assert s0 != s1 and g0[0] != g0[1] and g0 == g1   # distinct instances, agreed on by both


def test_job_throughput_counts_every_rank():
    f = 2.0e12
    assert bench.job_tflops(f, 1, 1000.0) == pytest.approx(2.0)
    assert bench.job_tflops(f, 4, 1000.0) == pytest.approx(8.0)
    assert bench.job_tflops(f, 4, 2000.0) == pytest.approx(4.0)
