"""Host logic of the multi-GPU paths on CPU with gloo: the benchmark's (each
rank draws its own workload instance, the slowest rank's time is what every
rank reports, the job throughput counts every rank's work) and the head-split
forward and backward of one problem (ranges, slices, the uneven all-gather),
with the single-GPU calls replaced by the fp64 oracle in the worker."""

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


def _sharded_worker(rank, world, port, out):
    import oracle
    from io_aware_exact_30_b200 import attn
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # stand-ins for the single-GPU calls (test doubles: no GPU here), which
        # also hold the ABI's rule that every pointer is 16-byte aligned
        def aligned(*xs):
            assert all(x.data_ptr() % 16 == 0 and x.is_contiguous() for x in xs)

        def fwd(q, k, v, causal, scale):
            aligned(q, k, v)
            o, lse = oracle.fwd(q.double().numpy(), k.double().numpy(), v.double().numpy(),
                                causal, scale)
            return torch.from_numpy(o).float(), torch.from_numpy(lse).float()

        def bwd(q, k, v, o, lse, do, causal, scale):
            aligned(q, k, v, o, lse, do)
            g = oracle.bwd(*(x.double().numpy() for x in (q, k, v, do)), causal, scale)
            return tuple(torch.from_numpy(x).float() for x in g)

        attn.forward, attn.backward = fwd, bwd
        B, H, N, d = 1, 5, 19, 64
        q, k, v, do = (torch.from_numpy(synth.tensor(3, st, (B, H, N, d), dtype="fp16")
                                        .astype(np.float32))
                       for st in (synth.STREAM_Q, synth.STREAM_K, synth.STREAM_V,
                                  synth.STREAM_DO))
        o, lse = attn.forward_sharded(q, k, v, True, 0.125)
        grads = attn.backward_sharded(q, k, v, o, lse, do, True, 0.125)
        o_part, lse_part, sn = attn.forward_sharded(q, k, v, True, 0.125, gather=False)
        out[rank] = (o.numpy(), lse.numpy(), [g.numpy() for g in grads], o_part.numpy(), sn)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_head_split_forward_and_backward(world):
    """Five heads over 2 or 3 ranks (uneven ranges): the gathered outputs equal
    the whole problem computed at once, on every rank."""
    import oracle
    from io_aware_exact_30_b200 import attn
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_sharded_worker, args=(world, port, out), nprocs=world,
                       start_method="spawn", join=True)
    B, H, N, d = 1, 5, 19, 64
    q, k, v, do = (synth.tensor(3, st, (B, H, N, d), dtype="fp16").astype(np.float64)
                   for st in (synth.STREAM_Q, synth.STREAM_K, synth.STREAM_V, synth.STREAM_DO))
    o_ref, lse_ref = oracle.fwd(q, k, v, True, 0.125)
    g_ref = oracle.bwd(q, k, v, do, True, 0.125)
    for r in range(world):
        o, lse, grads, o_part, (s, n) = out[r]
        assert (s, n) == attn.head_shard(B * H, r, world)
        np.testing.assert_allclose(o, o_ref, rtol=1e-6, atol=1e-6)
        np.testing.assert_allclose(lse, lse_ref, rtol=1e-6, atol=1e-6)
        for g, gr in zip(grads, g_ref):
            np.testing.assert_allclose(g, gr, rtol=1e-5, atol=1e-6)
        np.testing.assert_allclose(o_part[0], o_ref.reshape(B * H, N, d)[s:s + n],
                                   rtol=1e-6, atol=1e-6)


def test_head_shard_ranges():
    from io_aware_exact_30_b200 import attn
    for BH, W in ((64, 8), (12, 8), (5, 2), (3, 4), (0, 2), (1, 1)):
        sh = [attn.head_shard(BH, r, W) for r in range(W)]
        assert sum(n for _, n in sh) == BH
        assert sh[0][0] == 0 and all(a[0] + a[1] == b[0] for a, b in zip(sh, sh[1:]))
        assert max(n for _, n in sh) - min(n for _, n in sh) <= 1
    with pytest.raises(ValueError):
        attn.head_shard(4, 2, 2)
