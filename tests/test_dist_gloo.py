"""The multi-rank host logic of bench.py on CPU with gloo (world size 2).

The layer has no exchange step, so N GPUs either run N independent scenes of
the same size (replicas, weak scaling) or split one scene's heads (strong
scaling); the only collectives are the timing barrier and the max-over-ranks
reduction.  Here gloo ranks check that each replica rank gets its own scene
(same sizes, different values), that head-split ranks hold disjoint heads of
one scene that together cover it, that the reduction returns the slowest
rank's time on every rank, and the job value of both modes.
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


def _heads_worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        from synthetic import WORKLOADS, generate
        wl = bench.rank_workload(WORKLOADS["small"].with_(n_frames=2), rank, "heads")
        x = generate(wl)
        h0, h1 = bench.head_slice(world, rank, wl.n_heads)
        mine = x.q[:, h0:h1].float().sum(dim=(0, 2))  # per-head digests of this rank's slice
        full = x.q.float().sum(dim=(0, 2))
        my_ms = 20.0 + rank
        worst = bench.reduce_max(my_ms, dist, torch.device("cpu"))
        out[rank] = (h0, h1, mine.tolist(), full.tolist(), worst,
                     bench.job_value(world, wl.n_tokens, worst, "heads"), wl.n_tokens)
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(300)
@pytest.mark.parametrize("world", [2, 3])
def test_head_parallel_split(world):
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_heads_worker, args=(world, port, out), nprocs=world, join=True, start_method="spawn")
    covered = []
    for r in range(world):
        h0, h1, mine, full, worst, value, tokens = out[r]
        assert full == out[0][3], "every rank holds the same scene"
        assert mine == full[h0:h1]
        covered += list(range(h0, h1))
        assert worst == 20.0 + (world - 1)
        assert value == pytest.approx(tokens / (worst / 1e3)), "one scene's tokens over the slowest rank"
    assert covered == list(range(16)), "the ranks' heads are disjoint and cover all 16"
