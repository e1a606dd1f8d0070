"""The bench's multi-GPU logic on CPU: two gloo ranks, no GPU.

With N GPUs every rank runs its own sequence (independent problems, no data-path
collective); the job's time is the slowest rank's, taken with one all-reduce of a
scalar, and the job's throughput counts every rank's tokens.
"""
import dataclasses
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


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        from long_context_compressed_gated_b200 import inputs
        ms = bench.max_over_ranks(10.0 + 5.0 * rank, True, device="cpu")
        wl = dataclasses.replace(inputs.TINY, T=64)
        d = inputs.prefill_layer(wl, seed=bench.rank_seed(wl, rank))
        digest = float(d["K"].float().sum())
        digests = [None] * world
        dist.all_gather_object(digests, digest)
        out.put((rank, ms, digests, bench.job_throughput(wl.T, world, ms)))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_time_max_and_independent_inputs():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    res = [out.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    for rank, ms, digests, tput in res:
        assert ms == 15.0                      # the slowest rank's time on every rank
        assert digests[0] != digests[1]        # each rank has its own sequence
        assert tput == pytest.approx(64 * world / 15.0e-3)


def test_single_rank_helpers():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, False) == 3.5
    assert bench.job_throughput(32768, 1, 10.0) == pytest.approx(3.2768e6)
