"""The multi-process path of bench.py on CPU: two gloo ranks, each with its
own timing, agree on the max over ranks, and the whole-job throughput counts
every rank's work against the slowest rank's time (weak scaling, replicas
with no data-path collective)."""
import os
import socket

import pytest
import torch.multiprocessing as mp

from conftest import ROOT


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, results):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench
    d = bench.Dist()
    d.init("gloo")
    d.barrier()
    local_ms = 10.0 + 5.0 * rank          # rank 1 is the slow one
    ms = d.max(local_ms, "cpu")
    value = bench.job_throughput(1000.0, d.world, ms)
    results[rank] = (d.rank, d.world, ms, value)
    d.close()


@pytest.mark.timeout(120)
def test_two_gloo_ranks_agree_on_max_and_job_throughput():
    world = 2
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    results = manager.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, results)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(90)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    for r in range(world):
        rank, w, ms, value = results[r]
        assert rank == r and w == world
        assert ms == 15.0                         # the slowest rank's time on every rank
        assert value == pytest.approx(2 * 1000.0 / 0.015)


def test_single_process_needs_no_process_group():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    env = {k: os.environ.pop(k) for k in ("WORLD_SIZE", "RANK") if k in os.environ}
    try:
        d = bench.Dist()
        d.init("gloo")
        assert d.pg is None and d.max(3.5, "cpu") == 3.5
        assert bench.job_throughput(10.0, 1, 2.0) == pytest.approx(5000.0)
    finally:
        os.environ.update(env)
