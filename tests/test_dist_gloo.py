"""The multi-rank host logic of bench.py on CPU with gloo (world size 2).

The layer has no exchange step, so N GPUs run N independent scenes of the
same size; the only collectives are the timing barrier and the max-over-ranks
reduction.  Here two gloo ranks check that each rank gets its own scene (same
sizes, different values), that the reduction returns the slowest rank's time
on every rank, and that the job value counts every rank's tokens.
"""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        from synthetic import WORKLOADS, generate
        wl = bench.rank_workload(WORKLOADS["tiny"], rank)
        x = generate(wl)
        digest = float(x.q.float().sum())
        my_ms = 10.0 + 5.0 * rank
        dist.barrier()
        worst = bench.reduce_max(my_ms, dist, torch.device("cpu"))
        digests = [None] * world
        dist.all_gather_object(digests, (wl.n_tokens, digest))
        out[rank] = (worst, bench.job_value(world, wl.n_tokens, worst), digests)
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(300)
def test_two_rank_replicas_and_max_timing():
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, join=True, start_method="spawn")
    for r in range(world):
        worst, value, digests = out[r]
        assert worst == 15.0
        assert value == pytest.approx(2 * 512 / 0.015)
        sizes = {d[0] for d in digests}
        assert sizes == {512}
        assert digests[0][1] != digests[1][1], "ranks must run independent scenes"
