"""Host logic of the multi-GPU bench path, on CPU with two gloo ranks.

The decode path shards by sequences (each rank owns its own batch, no
data-path collective); the only cross-rank steps are the barriers and the
max-over-ranks timing that turns per-rank times into a whole-job rate.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, times, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        dist.barrier()
        slowest = bench.max_over_ranks(times[rank], torch.device("cpu"))
        out[rank] = slowest
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_max_over_ranks_and_rate(world):
    times = [12.5, 17.25]
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, times, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert [out[r] for r in range(world)] == [max(times)] * world
    # every rank decodes its own batch: the job rate counts all ranks' tokens against the slowest rank
    assert bench.whole_job_rate(world, 16, 100, max(times)) == pytest.approx(2 * 16 * 100 / 0.01725)


def test_single_process_is_identity():
    assert bench.max_over_ranks(3.0, torch.device("cpu")) == 3.0
    assert bench.whole_job_rate(1, 16, 10, 1.0) == pytest.approx(160000.0)
